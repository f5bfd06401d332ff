// router.cu -- router scoring, top-k selection and softmax renormalisation.
//
// The router scores each token against every expert and keeps the top_k
// ("Strata open-source runtime", section "the model itself": 10 of 512 per
// layer).  logits[t][e] = sum_i x[t][i] Wr[e][i] + b[e] in fp32; selection is
// largest first with equal logits going to the lower expert index and NaN last;
// the weights are the softmax of the selected logits.
//
// Small T (decode, verify windows): one warp per expert row streams Wr with
// 128-bit loads (the 4 MiB fp32 router is a sizeable part of a 1-token layer's
// bytes); the last CTA to finish (atomic counter in the workspace, reset by
// that CTA) runs the selection for the window.
// Large T (prefill): a tiled fp32 GEMM writes the logits, then one warp per
// token selects.
#include "internal.h"
#include "select.cuh"

namespace moe {

// ------------------------------------------------------------- small T router
// grid: ceil(E/4) CTAs of 16 warps; four warps per expert row, each a quarter
// of d.  The CTA's four rows of Wr (contiguous) are requested with one bulk
// async copy before the grid waits on its predecessor (Wr depends on nothing
// earlier), so the whole 4 MiB router is in flight at once.  The last CTA to
// finish (atomic counter in the workspace, reset by that CTA) selects.
// smem: 4*d fp32 (rows) | T*d bf16 (tokens) | 4*4*8 partial sums.
constexpr int kRouterRows = 4;
constexpr int kRouterWarps = 16;
__global__ void __launch_bounds__(kRouterWarps * 32) router_small_kernel(
    LayerDev L, const uint16_t* __restrict__ x, int T, uint32_t flags, float* __restrict__ logits,
    int32_t* __restrict__ ids, float* __restrict__ wout, Control* ctl) {
  extern __shared__ __align__(128) unsigned char smem[];
  float* wrs = reinterpret_cast<float*>(smem);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + (size_t)kRouterRows * L.d * 4);
  __shared__ float red[kMaxDecodeT];
  __shared__ float part[kRouterRows][4][kMaxDecodeT];
  __shared__ int s_last;
  __shared__ __align__(8) uint64_t bar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = blockIdx.x * kRouterRows;
  const int nrows = min(kRouterRows, L.E - e0);
  const int row = warp >> 2, quarter = warp & 3;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    const uint32_t bytes = (uint32_t)nrows * L.d * 4;
    mbar_arrive_expect_tx(&bar, bytes);
    bulk_g2s(wrs, L.Wr + (size_t)e0 * L.d, bytes, &bar);
  }
  pdl_wait();
  pdl_launch_dependents();
  stage_tokens(x, T, L.d, flags & MOE_F_PRENORM, xs, red);   // ends with __syncthreads
  const bool have = mbar_wait(&bar, 0, ctl, 0x110);

  if (row < nrows && have) {
    float acc[kMaxDecodeT];
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) acc[t] = 0.f;
    const float4* wr = reinterpret_cast<const float4*>(wrs + (size_t)row * L.d);
    const int nc = L.d / 4, c0 = quarter * (nc / 4), c1 = c0 + nc / 4;
#pragma unroll 4
    for (int c = c0 + lane; c < c1; c += 32) {
      const float4 wv = wr[c];
#pragma unroll
      for (int t = 0; t < kMaxDecodeT; ++t) {
        if (t < T) {
          const uint2 xv = *reinterpret_cast<const uint2*>(xs + t * L.d + 4 * c);
          acc[t] = fmaf(__uint_as_float(xv.x << 16), wv.x, acc[t]);
          acc[t] = fmaf(__uint_as_float(xv.x & 0xFFFF0000u), wv.y, acc[t]);
          acc[t] = fmaf(__uint_as_float(xv.y << 16), wv.z, acc[t]);
          acc[t] = fmaf(__uint_as_float(xv.y & 0xFFFF0000u), wv.w, acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) {
      if (t < T) {
        const float s = warp_sum(acc[t]);
        if (lane == 0) part[row][quarter][t] = s;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < nrows * T) {
    const int r = threadIdx.x / T, t = threadIdx.x % T, e = e0 + r;
    const float s = part[r][0][t] + part[r][1][t] + part[r][2][t] + part[r][3][t];
    logits[(size_t)t * L.E + e] = s + (L.bias ? L.bias[e] : 0.f);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();   // release this CTA's logits
    const uint32_t old = atomicAdd(&ctl->router_done, 1u);
    s_last = (old == gridDim.x - 1);
    if (s_last) __threadfence();   // acquire every CTA's logits; the barrier below publishes
  }
  __syncthreads();
  if (!s_last) return;
  for (int t = warp; t < T; t += kRouterWarps)
    warp_topk(logits + (size_t)t * L.E, L.pref, L.counts, L.E, L.k, ids + (size_t)t * L.k, wout + (size_t)t * L.k,
              ctl, flags & MOE_F_DEBUG);
  if (threadIdx.x == 0) atomicExch(&ctl->router_done, 0u);
}

size_t router_small_smem(int d, int T) {
  return (size_t)kRouterRows * d * 4 + ((size_t)T * d * 2 + 15) / 16 * 16;
}

cudaError_t launch_router_small(const LayerDev& L, const uint16_t* x, int T, uint32_t flags,
                                float* logits, int32_t* ids, float* w, Control* ctl,
                                cudaStream_t st) {
  const size_t smem = router_small_smem(L.d, T);
  cudaError_t e = cudaFuncSetAttribute(router_small_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((L.E + kRouterRows - 1) / kRouterRows);
  return launch_pdl(router_small_kernel, grid, dim3(kRouterWarps * 32), smem, st, L, x, T, flags,
                    logits, ids, w, ctl);
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
  // the lean rescan: fewer registers, more warps of this batch kernel resident
  warp_topk<true>(logits + (size_t)t * L.E, L.pref, L.counts, L.E, L.k, ids + (size_t)t * L.k, w + (size_t)t * L.k, ctl,
            flags & MOE_F_DEBUG);
}

cudaError_t launch_router_large(const LayerDev& L, const uint16_t* x, int T, uint32_t flags,
                                float* logits, int32_t* ids, float* w, uint16_t* wsplit,
                                Control* ctl, cudaStream_t st) {
  // the caller's split router weights when given, else split into the workspace
  uint16_t* hi = L.wsplit ? const_cast<uint16_t*>(L.wsplit) : wsplit;
  cudaError_t e = launch_router_tc(L, x, T, logits, hi, hi + (size_t)L.E * L.d, !L.wsplit, ctl, st);
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
