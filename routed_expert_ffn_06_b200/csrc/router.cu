// router.cu -- router scoring, top-k selection and softmax renormalisation.
//
// The router scores each token against every expert and keeps the top_k
// ("Strata open-source runtime", section "the model itself": 10 of 512 per
// layer).  logits[t][e] = sum_i x[t][i] Wr[e][i] + b[e] in fp32; selection is
// largest first with equal logits going to the lower expert index and NaN last;
// the weights are the softmax of the selected logits.
//
// Small T (decode, verify windows): one warp per expert row holds its row of
// Wr in registers (the 4 MiB fp32 router is a sizeable part of a 1-token
// layer's bytes) and writes the logits; the expert kernel that follows selects
// (or, for moe_route_topk, a one-warp-per-token selection kernel).
// Large T (prefill): a tiled fp32 GEMM writes the logits, then one warp per
// token selects.
#include "internal.h"
#include "select.cuh"

namespace moe {

// ------------------------------------------------------------ decode router
// One warp per expert row, four rows per CTA.  Each lane keeps its share of
// the row (d / 128 float4, up to NPRE of them) in registers, loaded before the
// kernel waits for its predecessor: the router weights do not depend on it, so
// their 4 MiB stream while the previous layer finishes.  After the wait the
// warp reads the window's tokens (optionally RMS-normalised: the sum of squares
// in the same fixed order as the expert kernel's), forms the T dot products
// and writes the logits.  Selection happens where the logits are consumed.
// At most 88 registers per thread, so that it fits beside an expert CTA and a
// combine CTA of the previous window on one SM.
constexpr int kGemvWarps = 4;
template <int NPRE>
__global__ void __maxnreg__(88) router_gemv_kernel(
    const __grid_constant__ LayerDev L, const uint16_t* __restrict__ x, int T, uint32_t flags, float* __restrict__ logits,
    unsigned char* __restrict__ xfrag, Control* ctl) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kGemvWarps + warp;
  const int d = L.d, nc4 = d / 4;
  const bool have = logits != nullptr && e < L.E;
  const float4* wr = reinterpret_cast<const float4*>(L.Wr + (size_t)(have ? e : 0) * d);
  float4 w[NPRE];
#pragma unroll
  for (int j = 0; j < NPRE; ++j) {
    const int c = lane + 32 * j;
    w[j] = (have && c < nc4) ? ldg_nc_f4(wr + c) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // x may come from the grid this one waits for: read it only afterwards, and
  // let the next grid (which reads x before its own wait) start only then
  pdl_wait();
  pdl_launch_dependents();
  const bool pn = flags & MOE_F_PRENORM;
  // 1 / RMS of token t (the sum of squares in the expert kernel's fixed order)
  auto inv_rms = [&](int t) {
    float ss = 0.f;
#pragma unroll 1
    for (int i = lane * 8; i < d; i += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(x + (size_t)t * d + i);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = __uint_as_float(w4[q] << 16), b = __uint_as_float(w4[q] & 0xFFFF0000u);
        ss += a * a + b * b;
      }
    }
    return rsqrtf(warp_sum(ss) / (float)d + kRmsEps);
  };
  // The expert kernel's operands for the window's tokens: per (quantisation
  // group c, token n) the 32 values as the mma B fragments of lanes 4n..4n+3
  // (fp16; 2-bit: value / 4^m for columns 8m..8m+7, the offset form) and, for
  // 2-bit, the correction sum of B * (1024 + 2 * 4^m).  One warp per (c, n),
  // lane q < 16 holding columns 2q, 2q+1.  fp16 operands: values outside the
  // fp16 range are flagged (always on).
  if (xfrag) {
    const int nG = d / kGroup, npairs = kMaxDecodeT * nG;
    uint32_t* xs = reinterpret_cast<uint32_t*>(xfrag);
    float* corr = reinterpret_cast<float*>(xfrag + (size_t)nG * 32 * 16);
    bool bad = false;
#pragma unroll 1
    for (int p = blockIdx.x * kGemvWarps + warp; p < npairs; p += gridDim.x * kGemvWarps) {
      const int c = p >> 3, n = p & 7, m = (lane >> 2) & 3;
      const float inv = (pn && n < T) ? inv_rms(n) : 1.f;
      float v0 = 0.f, v1 = 0.f;
      if (lane < 16 && n < T) {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(x + (size_t)n * d + 32 * c + 2 * lane);
        v0 = __uint_as_float(u << 16);
        v1 = __uint_as_float(u & 0xFFFF0000u);
        if (pn) {
          v0 = __bfloat162float(__float2bfloat16_rn(v0 * inv));
          v1 = __bfloat162float(__float2bfloat16_rn(v1 * inv));
        }
        bad |= !(fabsf(v0) <= 65504.f) || !(fabsf(v1) <= 65504.f);
      }
      float cs = 0.f;
      __half2 bh;
      if (L.bits == 2) {
        const float sc = 1.f / (float)(1 << (2 * m));
        bh = __floats2half2_rn(v0 * sc, v1 * sc);
        cs = (__low2float(bh) + __high2float(bh)) * (1024.f + 2.f * (float)(1 << (2 * m)));
      } else {
        bh = __floats2half2_rn(v0, v1);
      }
      if (lane < 16) xs[((size_t)(c * 32 + n * 4 + (lane & 3))) * 4 + m] = h2_as_u32(bh);
      cs = warp_sum(lane < 16 ? cs : 0.f);
      if (lane == 0) corr[c * kMaxDecodeT + n] = cs;
    }
    if (bad) record_error(ctl, kErrNonFinite, 0x120);
  }
  if (!have) return;
  const float b = L.bias ? L.bias[e] : 0.f;
  // two tokens per pass: twice the loads in flight per memory round trip
#pragma unroll 1
  for (int t = 0; t < T; t += 2) {
    const bool two = t + 1 < T;
    const float inv0 = pn ? inv_rms(t) : 1.f;
    const float inv1 = (pn && two) ? inv_rms(t + 1) : 1.f;
    const uint16_t* x0 = x + (size_t)t * d;
    const uint16_t* x1 = two ? x0 + d : x0;
    auto dot4 = [&](float acc, const float4& wv, const uint16_t* xt, float inv, int c) {
      const uint2 u = *reinterpret_cast<const uint2*>(xt + 4 * c);
      float v[4] = {__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                    __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u)};
      if (pn) {
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = __bfloat162float(__float2bfloat16_rn(v[q] * inv));
      }
      acc = fmaf(v[0], wv.x, acc);
      acc = fmaf(v[1], wv.y, acc);
      acc = fmaf(v[2], wv.z, acc);
      return fmaf(v[3], wv.w, acc);
    };
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < NPRE; ++j) {
      const int c = lane + 32 * j;
      if (c < nc4) {
        a0 = dot4(a0, w[j], x0, inv0, c);
        a1 = dot4(a1, w[j], x1, inv1, c);
      }
    }
#pragma unroll 1
    for (int c = lane + 32 * NPRE; c < nc4; c += 32) {
      const float4 wv = ldg_nc_f4(wr + c);
      a0 = dot4(a0, wv, x0, inv0, c);
      a1 = dot4(a1, wv, x1, inv1, c);
    }
    a0 = warp_sum(a0);
    a1 = warp_sum(a1);
    if (lane == 0) {
      logits[(size_t)t * L.E + e] = a0 + b;
      if (two) logits[(size_t)(t + 1) * L.E + e] = a1 + b;
    }
  }
}

cudaError_t launch_router_gemv(const LayerDev& L, const uint16_t* x, int T, uint32_t flags,
                               float* logits, unsigned char* xfrag, Control* ctl,
                               cudaStream_t st) {
  // logits: one warp per expert row; token fragments only: enough warps for
  // the (group, token) pairs
  const int rows = logits ? L.E : 0;
  const int pairs = xfrag ? kMaxDecodeT * (L.d / kGroup) : 0;
  const int warps = rows > pairs ? rows : pairs;
  const dim3 grid((warps + kGemvWarps - 1) / kGemvWarps);
  return launch_pdl(router_gemv_kernel<16>, grid, dim3(kGemvWarps * 32), 0, st, L, x, T, flags,
                    logits, xfrag, ctl);
}

// ------------------------------------------------------------ prefill router
// RMSNorm (optional) of every token into xn (bf16) and an fp16 copy x16 of the
// block input for the expert GEMMs.  One warp per token.
__global__ void __launch_bounds__(256) prep_tokens_kernel(const uint16_t* __restrict__ x, int T,
                                                          int d, uint32_t flags,
                                                          uint16_t* __restrict__ xn,
                                                          __half* __restrict__ x16, Control* ctl) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= T) return;
  const uint16_t* xr = x + (size_t)warp * d;
  float inv = 1.f;
  if (flags & MOE_F_PRENORM) {
    float ss = 0.f;
    for (int i = lane; i < d; i += 32) {
      float v = bf16_bits_to_float(xr[i]);
      ss += v * v;
    }
    ss = warp_sum(ss);
    inv = rsqrtf(ss / (float)d + kRmsEps);
  }
  // fp16 operands: values outside the fp16 range are flagged (always on)
  bool bad = false;
  for (int i = lane; i < d; i += 32) {
    float v = bf16_bits_to_float(xr[i]);
    if (flags & MOE_F_PRENORM) {
      __nv_bfloat16 bv = __float2bfloat16_rn(v * inv);
      uint16_t bb = *reinterpret_cast<uint16_t*>(&bv);
      xn[(size_t)warp * d + i] = bb;
      v = bf16_bits_to_float(bb);
    }
    bad |= !(fabsf(v) <= 65504.f);
    x16[(size_t)warp * d + i] = __float2half_rn(v);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(ctl, kErrNonFinite, 0x200);
}

__global__ void __launch_bounds__(256) topk_kernel(LayerDev L, const float* __restrict__ logits,
                                                   int T, int32_t* __restrict__ ids,
                                                   float* __restrict__ w, uint32_t flags,
                                                   Control* ctl) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  warp_topk(logits + (size_t)t * L.E, L.E, L.k, ids + (size_t)t * L.k, w + (size_t)t * L.k, ctl,
            flags & MOE_F_DEBUG);
}

cudaError_t launch_topk(const LayerDev& L, const float* logits, int T, int32_t* ids, float* w,
                        uint32_t flags, Control* ctl, cudaStream_t st) {
  return launch_pdl(topk_kernel, dim3((T + 7) / 8), dim3(256), 0, st, L, logits, T, ids, w, flags,
                    ctl);
}

cudaError_t launch_router_large(const LayerDev& L, const uint16_t* x, int T, uint32_t flags,
                                float* logits, int32_t* ids, float* w, uint16_t* wsplit,
                                Control* ctl, cudaStream_t st) {
  cudaError_t e = launch_router_tc(L, x, T, logits, wsplit, wsplit + (size_t)L.E * L.d, ctl, st);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_kernel, dim3((T + 7) / 8), dim3(256), 0, st, L,
                    static_cast<const float*>(logits), T, ids, w, flags, ctl);
}

cudaError_t launch_prep_tokens(const uint16_t* x, int T, int d, uint32_t flags, uint16_t* xn,
                               __half* x16, Control* ctl, cudaStream_t st) {
  return launch_pdl(prep_tokens_kernel, dim3((T + 7) / 8), dim3(256), 0, st, x, T, d, flags, xn,
                    x16, ctl);
}

}  // namespace moe
