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

namespace moe {

constexpr float kRmsEps = 1e-6f;

// ---------------------------------------------------------------- selection
// One warp selects top_k of E (E <= 1024) logits of one token and writes the
// ids (largest first) and renormalised weights.
__device__ void warp_topk(const float* __restrict__ row, int E, int k, int32_t* __restrict__ ids,
                          float* __restrict__ w, Control* ctl, bool debug) {
  const int lane = threadIdx.x & 31;
  uint32_t key[32];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    int e = lane + 32 * i;
    key[i] = 0u;
    if (e < E) {
      float v = __ldcg(row + e);
      if (debug && !isfinite(v)) record_error(ctl, kErrNonFinite, 0x100);
      key[i] = order_key(v);
    }
  }
  float my_v = 0.f;
  for (int j = 0; j < k; ++j) {
    // lane-local best: larger key, then lower index (lower i within a lane)
    unsigned long long best = 0ull;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u)) {
        unsigned long long c = (static_cast<unsigned long long>(key[i]) << 32) |
                               static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(e));
        best = c > best ? c : best;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    const uint32_t e = 0xFFFFFFFFu - static_cast<uint32_t>(best & 0xFFFFFFFFull);
    const uint32_t kk = static_cast<uint32_t>(best >> 32);
    if ((int)(e & 31u) == lane) taken |= 1u << (e >> 5);
    uint32_t u = (kk & 0x80000000u) ? (kk & 0x7FFFFFFFu) : ~kk;
    const float v = __uint_as_float(u);
    if (lane == j) my_v = v;
    if (lane == 0) ids[j] = static_cast<int32_t>(e);
  }
  const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = lane < k ? expf(my_v - v0) : 0.f;
  const float den = warp_sum(ex);
  if (lane < k) w[lane] = ex / den;
}

// --------------------------------------------------------- x (bf16) staging
// Loads T token rows into shared memory as bf16 bits; with PRENORM replaces
// them by bf16(x / sqrt(mean(x^2) + eps)), computed in fp32.
__device__ void stage_tokens(const uint16_t* __restrict__ x, int T, int d, bool prenorm,
                             uint16_t* xs, float* red) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int nw = nt / 32;
  for (int t = 0; t < T; ++t) {
    const uint16_t* xr = x + (size_t)t * d;
    float ss = 0.f;
    for (int i = tid; i < d; i += nt) {
      uint16_t b = xr[i];
      xs[t * d + i] = b;
      float v = bf16_bits_to_float(b);
      ss += v * v;
    }
    if (prenorm) {
      ss = warp_sum(ss);
      if ((tid & 31) == 0) red[tid >> 5] = ss;
      __syncthreads();
      float tot = 0.f;
      for (int i = 0; i < nw; ++i) tot += red[i];
      const float inv = rsqrtf(tot / (float)d + kRmsEps);
      for (int i = tid; i < d; i += nt) {
        float v = bf16_bits_to_float(xs[t * d + i]) * inv;
        __nv_bfloat16 bv = __float2bfloat16_rn(v);
        xs[t * d + i] = *reinterpret_cast<uint16_t*>(&bv);
      }
      __syncthreads();
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------- small T router
// grid: ceil(E/4) CTAs of 4 warps, one warp per expert row.
// smem: T*d bf16 + 32 floats.
__global__ void __launch_bounds__(128) router_small_kernel(LayerDev L, const uint16_t* __restrict__ x,
                                                           int T, uint32_t flags,
                                                           float* __restrict__ logits,
                                                           int32_t* __restrict__ ids,
                                                           float* __restrict__ wout, Control* ctl) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
  float* red = reinterpret_cast<float*>(smem + ((size_t)T * L.d * 2 + 15) / 16 * 16);
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 4 + warp;

  // Wr does not depend on earlier kernels: pull this warp's row into L2 first.
  if (e < L.E && lane == 0) {
    const char* row = reinterpret_cast<const char*>(L.Wr + (size_t)e * L.d);
    for (int off = 0; off < L.d * 4; off += 4096) {
      int n = min(4096, L.d * 4 - off);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(row + off), "r"(n) : "memory");
    }
  }
  pdl_wait();
  pdl_launch_dependents();
  stage_tokens(x, T, L.d, flags & MOE_F_PRENORM, xs, red);

  if (e < L.E) {
    float acc[kMaxDecodeT];
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) acc[t] = 0.f;
    const float4* wr = reinterpret_cast<const float4*>(L.Wr + (size_t)e * L.d);
    const int nc = L.d / 4;
    for (int c = lane; c < nc; c += 32) {
      const float4 wv = __ldg(wr + c);
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
    const float b = L.bias ? L.bias[e] : 0.f;
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) {
      if (t < T) {
        float s = warp_sum(acc[t]);
        if (lane == 0) logits[(size_t)t * L.E + e] = s + b;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(&ctl->router_done, 1u);
    s_last = (old == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int t = warp; t < T; t += 4)
    warp_topk(logits + (size_t)t * L.E, L.E, L.k, ids + (size_t)t * L.k, wout + (size_t)t * L.k,
              ctl, flags & MOE_F_DEBUG);
  if (threadIdx.x == 0) atomicExch(&ctl->router_done, 0u);
}

cudaError_t launch_router_small(const LayerDev& L, const uint16_t* x, int T, uint32_t flags,
                                float* logits, int32_t* ids, float* w, Control* ctl,
                                cudaStream_t st) {
  size_t smem = ((size_t)T * L.d * 2 + 15) / 16 * 16 + 32 * sizeof(float);
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(router_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         96 * 1024);
    attr_done = true;
  }
  dim3 grid((L.E + 3) / 4);
  return launch_pdl(router_small_kernel, grid, dim3(128), smem, st, L, x, T, flags, logits, ids,
                    w, ctl);
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
  for (int i = lane; i < d; i += 32) {
    float v = bf16_bits_to_float(xr[i]);
    if (flags & MOE_F_PRENORM) {
      __nv_bfloat16 bv = __float2bfloat16_rn(v * inv);
      uint16_t bb = *reinterpret_cast<uint16_t*>(&bv);
      xn[(size_t)warp * d + i] = bb;
      v = bf16_bits_to_float(bb);
    }
    if ((flags & MOE_F_DEBUG) && !(fabsf(v) <= 65504.f)) record_error(ctl, kErrNonFinite, 0x200);
    x16[(size_t)warp * d + i] = __float2half_rn(v);
  }
}

// fp32 GEMM: logits[T][E] = X[T][d] (bf16) * Wr[E][d]^T + b.
// 128 x 128 tile, K-step 16, 256 threads, 8 x 8 outputs per thread.
constexpr int RB_M = 128, RB_N = 128, RB_K = 16;
__global__ void __launch_bounds__(256) router_gemm_kernel(LayerDev L, const uint16_t* __restrict__ X,
                                                          int T, float* __restrict__ logits) {
  __shared__ __align__(16) float As[RB_K][RB_M + 4];
  __shared__ __align__(16) float Bs[RB_K][RB_N + 4];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * RB_M, n0 = blockIdx.x * RB_N;
  const int tx = tid % 16, ty = tid / 16;   // 16 x 16 threads; rows ty+16i, cols tx+16j
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  const int d = L.d;
  for (int k0 = 0; k0 < d; k0 += RB_K) {
    // A tile: 128 rows x 16 k (bf16) -> As[k][m]
    for (int i = tid; i < RB_M * RB_K; i += 256) {
      int m = i / RB_K, kk = i % RB_K;
      int gm = m0 + m;
      float v = 0.f;
      if (gm < T) v = bf16_bits_to_float(X[(size_t)gm * d + k0 + kk]);
      As[kk][m] = v;
    }
    // B tile: 128 experts x 16 k (fp32) -> Bs[k][n]
    for (int i = tid; i < RB_N * RB_K; i += 256) {
      int n = i / RB_K, kk = i % RB_K;
      int gn = n0 + n;
      Bs[kk][n] = gn < L.E ? __ldg(L.Wr + (size_t)gn * d + k0 + kk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < RB_K; ++kk) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int gm = m0 + ty + 16 * i;
    if (gm >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      int gn = n0 + tx + 16 * j;
      if (gn < L.E) logits[(size_t)gm * L.E + gn] = acc[i][j] + (L.bias ? L.bias[gn] : 0.f);
    }
  }
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

cudaError_t launch_router_large(const LayerDev& L, const uint16_t* x, int T, uint32_t flags,
                                float* logits, int32_t* ids, float* w, Control* ctl,
                                cudaStream_t st) {
  dim3 grid((L.E + RB_N - 1) / RB_N, (T + RB_M - 1) / RB_M);
  cudaError_t e = launch_pdl(router_gemm_kernel, grid, dim3(256), 0, st, L, x, T, logits);
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
