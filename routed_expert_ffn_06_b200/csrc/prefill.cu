// prefill.cu -- prefill expert step (placeholder until the grouped GEMM lands).
#include "internal.h"

namespace moe {

size_t prefill_ws_bytes(const LayerDev& L, int T, size_t* parts) {
  const int Fmax = L.F > L.Fs ? L.F : L.Fs;
  const size_t nblk = ((size_t)T + 255) / 256;
  parts[0] = (size_t)T * L.d * 2;
  parts[1] = (size_t)T * L.d * 2;
  parts[2] = (size_t)(L.E + 1) * 4;
  parts[3] = (size_t)(L.E + 2) * 4;
  parts[4] = (size_t)T * L.k * 4;
  parts[5] = nblk * L.E * 4;
  parts[6] = 16;
  parts[7] = ((size_t)T * L.k + T + (size_t)(L.E + 1) * 128) * Fmax * 2;
  parts[8] = (size_t)T * L.d * 4;
  size_t tot = 0;
  for (int i = 0; i < 9; ++i) tot += parts[i];
  return tot;
}

cudaError_t launch_prefill(const LayerDev&, const uint16_t*, int, const int32_t*, const float*,
                           uint16_t*, int32_t*, int32_t*, uint32_t, char*, const WsLayout&,
                           cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace moe
