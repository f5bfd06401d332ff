// pack.cu -- host-side quantiser and packer for expert weights (moe_pack.h).
// Host code only: it runs on the CPU and touches no device.
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include "moe_pack.h"

namespace {

constexpr int kGroupSize = 32;
constexpr int kRows = 16;   // rows per tile

// One group: fp16 scale bits and the 32 codes.
void quantise_group(const float* w, int bits, uint16_t* scale_out, uint8_t* q) {
  const int off = 1 << (bits - 1), qmax = (1 << bits) - 1;
  float m = w[0];
  for (int j = 1; j < kGroupSize; ++j)
    if (fabsf(w[j]) > fabsf(m)) m = w[j];
  const __half s16 = __float2half_rn(m / (float)(-off));
  const float s = __half2float(s16);
  *scale_out = __half_as_ushort(s16);
  for (int j = 0; j < kGroupSize; ++j) {
    if (s == 0.f) {
      q[j] = (uint8_t)off;
      continue;
    }
    float v = nearbyintf(w[j] / s) + (float)off;   // round half to even
    v = v < 0.f ? 0.f : (v > (float)qmax ? (float)qmax : v);
    q[j] = (uint8_t)v;
  }
}

}  // namespace

extern "C" moe_status moe_pack_host(const float* w, int32_t rows, int32_t cols, int32_t bits,
                                    uint8_t* codes, uint16_t* scales) {
  if (!w || !codes || !scales) return MOE_ERR_INVALID_ARG;
  if (rows <= 0 || rows % kRows || cols <= 0 || cols % kGroupSize || (bits != 2 && bits != 3))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  const int nG = cols / kGroupSize;
  const size_t lo_bytes = (size_t)nG * kRows * 8, hi_bytes = bits == 3 ? (size_t)nG * kRows * 4 : 0;
  const size_t tile_bytes = lo_bytes + hi_bytes;
  for (int tile = 0; tile < rows / kRows; ++tile) {
    uint8_t* tc = codes + (size_t)tile * tile_bytes;
    uint16_t* ts = scales + (size_t)tile * nG * kRows;
    memset(tc, 0, tile_bytes);
    for (int r = 0; r < kRows; ++r) {
      const float* row = w + (size_t)(tile * kRows + r) * cols;
      for (int c = 0; c < nG; ++c) {
        uint8_t q[kGroupSize];
        quantise_group(row + c * kGroupSize, bits, &ts[c * kRows + r], q);
        // word (c, r): code j = 8m + 2t + h -> low two bits at bit 32h + 8t + 2m
        // of the 8-byte word, high bit (3-bit) at bit 16h + 4t + m of the 4-byte word
        uint8_t* lo = tc + ((size_t)c * kRows + r) * 8;
        uint8_t* hi = tc + lo_bytes + ((size_t)c * kRows + r) * 4;
        for (int j = 0; j < kGroupSize; ++j) {
          const int m = j >> 3, t = (j >> 1) & 3, h = j & 1;
          const int pl = 32 * h + 8 * t + 2 * m;
          lo[pl >> 3] |= (uint8_t)((q[j] & 3) << (pl & 7));
          if (bits == 3) {
            const int ph = 16 * h + 4 * t + m;
            hi[ph >> 3] |= (uint8_t)(((q[j] >> 2) & 1) << (ph & 7));
          }
        }
      }
    }
  }
  return MOE_OK;
}
