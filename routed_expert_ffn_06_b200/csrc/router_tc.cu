// router_tc.cu -- router logits of a long token batch on the tensor cores.
//
// logits[t][e] = sum_i x[t][i] * Wr[e][i] + b[e]: the router of the routed
// block ("Why Strata is fast on low-VRAM GPUs", the MoE paragraph: each token
// scores all 512 experts and keeps 10).  x is bf16 and enters the MMA exactly;
// the fp32 router weights are split into two bf16 terms, hi = bf16(Wr) and
// lo = bf16(Wr - hi), which leave a residual below 2^-16 |Wr|.  Both products
// accumulate in fp32 in TMEM, so a logit carries an error far below the
// 1e-4 * sum|x Wr| bound of an fp32 dot product in any order, while the
// contraction runs at tensor-core rate instead of the fp32 SIMT rate.
//
// One CTA computes a 128-expert x 128-token tile: warp 0 loads the hi, lo and
// token tiles of each 64-wide k-step by TMA (128-byte swizzle) into a 3-stage
// ring, one thread of warp 1 issues 2 x 4 tcgen05.mma (kind::f16, bf16
// operands) per k-step, and warps 2-5 read TMEM (lane = expert, column =
// token) and store the logits with the bias added.
#include <cuda.h>

#include "internal.h"
#include "tc.cuh"

namespace moe {

bool make_map_b16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows);

constexpr int RT_STAGES = 3;
constexpr int RT_TILE = 128 * 128;        // 128 rows x 64 bf16
constexpr int RT_STAGE = 3 * RT_TILE;     // hi, lo, tokens
constexpr int RT_THREADS = 6 * 32;

__global__ void __launch_bounds__(256) split_router_kernel(const float* __restrict__ Wr, long long n4,
                                                           uint2* __restrict__ hi,
                                                           uint2* __restrict__ lo) {
  pdl_wait();
  pdl_launch_dependents();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 w = reinterpret_cast<const float4*>(Wr)[i];
    const __nv_bfloat162 h01 = __floats2bfloat162_rn(w.x, w.y), h23 = __floats2bfloat162_rn(w.z, w.w);
    const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
    const __nv_bfloat162 l01 = __floats2bfloat162_rn(w.x - f01.x, w.y - f01.y);
    const __nv_bfloat162 l23 = __floats2bfloat162_rn(w.z - f23.x, w.w - f23.y);
    hi[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
    lo[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&l01), *reinterpret_cast<const uint32_t*>(&l23));
  }
}

struct alignas(64) RtMaps {
  CUtensorMap hi, lo, x;
};

__device__ __forceinline__ void rt_tma_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(RT_THREADS, 1) router_tc_kernel(const float* __restrict__ bias,
                                                                   int E, int T, int d,
                                                                   float* __restrict__ logits,
                                                                   Control* ctl,
                                                                   const __grid_constant__ RtMaps mp) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RT_STAGES * RT_STAGE);
  uint64_t* empty = full + RT_STAGES;
  uint64_t* done = empty + RT_STAGES;
  uint32_t* holder = reinterpret_cast<uint32_t*>(done + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int e0 = blockIdx.x * 128, t0 = blockIdx.y * 128;
  const int KS = (d + 63) / 64;   // a ragged last k-step reads zeros past d (TMA fill)

  if (tid == 0) {
    for (int s = 0; s < RT_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(holder, 128);
    tmem_relinquish();
  }
  if (warp == 0 && lane < 3) {
    const CUtensorMap* maps[3] = {&mp.hi, &mp.lo, &mp.x};
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(maps[lane])) : "memory");
  }
  pdl_wait();
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  bool ok = true;

  // A role whose bounded wait runs out stops issuing; before the CTA ends, the
  // loader waits for the copies it issued and the MMA lane for its MMAs.
  if (warp == 0) {
    if (lane == 0) {
      int s = 0, ks = 0;
      uint32_t ph = 0;
      for (; ks < KS; ++ks) {
        if (ks >= RT_STAGES && !mbar_wait(&empty[s], ph ^ 1u, ctl, 0x250)) break;
        unsigned char* st = smem + s * RT_STAGE;
        mbar_arrive_expect_tx(&full[s], RT_STAGE);
        rt_tma_2d(st, &mp.hi, 64 * ks, e0, &full[s]);
        rt_tma_2d(st + RT_TILE, &mp.lo, 64 * ks, e0, &full[s]);
        rt_tma_2d(st + 2 * RT_TILE, &mp.x, 64 * ks, t0, &full[s]);
        if (++s == RT_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      // the newest phase of each stage may be unconsumed: its copies land first
      for (int j = ks > RT_STAGES ? ks - RT_STAGES : 0; j < ks; ++j)
        mbar_wait(&full[j % RT_STAGES], (uint32_t)(j / RT_STAGES) & 1u, ctl, 0x253);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // kind::f16 with bf16 A and B, fp32 D, M = N = 128, both K-major
      const uint32_t idesc = idesc_f16_f32(128, 128) | (1u << 7) | (1u << 10);
      const uint64_t desc0 = sw128_kmajor_desc(smem_u32(smem));
      int s = 0;
      uint32_t ph = 0;
      for (int ks = 0; ks < KS; ++ks) {
        if (!mbar_wait(&full[s], ph, ctl, 0x251)) break;
        tc_fence_after();
        const uint64_t ah = desc0 + (uint64_t)(s * (RT_STAGE >> 4));
        const uint64_t al = ah + (RT_TILE >> 4), bx = ah + 2 * (RT_TILE >> 4);
        tc_mma_f16(tmem, ah, bx, idesc, ks > 0 ? 1u : 0u);
        tc_mma_f16(tmem, ah + 2, bx + 2, idesc, 1u);
        tc_mma_f16(tmem, ah + 4, bx + 4, idesc, 1u);
        tc_mma_f16(tmem, ah + 6, bx + 6, idesc, 1u);
        tc_mma_f16(tmem, al, bx, idesc, 1u);
        tc_mma_f16(tmem, al + 2, bx + 2, idesc, 1u);
        tc_mma_f16(tmem, al + 4, bx + 4, idesc, 1u);
        tc_mma_f16(tmem, al + 6, bx + 6, idesc, 1u);
        tc_commit(&empty[s]);
        if (++s == RT_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      // done arrives once every MMA issued has completed (also after a
      // give-up); this lane releases the TMEM only after that
      tc_commit(done);
      mbar_wait(done, 0, ctl, 0x254);
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 = experts of those rows
    const int q = warp & 3;
    if (ok) ok = mbar_wait(done, 0, ctl, 0x252);
    tc_fence_after();
    const int e = e0 + 32 * q + lane;
    const float b = (bias && e < E) ? bias[e] : 0.f;
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
      tmem_ld_wait();
      if (ok && e < E) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = t0 + c0 + j;
          if (t < T) logits[(size_t)t * E + e] = __uint_as_float(v[j]) + b;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 128);
}

size_t router_tc_smem() { return (size_t)RT_STAGES * RT_STAGE + 2 * RT_STAGES * 8 + 8 + 16 + 1024; }

// hi/lo: workspace [E][d] bf16 each.  x: bf16 [T][d] (16-byte aligned).
cudaError_t launch_split_router(const float* Wr, int E, int d, uint16_t* hi, uint16_t* lo,
                                cudaStream_t st) {
  const long long n4 = (long long)E * d / 4;
  int g = (int)((n4 + 255) / 256);
  if (g > 2 * sm_count()) g = 2 * sm_count();
  return launch_pdl(split_router_kernel, dim3(g), dim3(256), 0, st, Wr, n4,
                    reinterpret_cast<uint2*>(hi), reinterpret_cast<uint2*>(lo));
}

// hi/lo: [E][d] bf16 each; split = true writes them from Wr first (otherwise
// they hold the split already).
cudaError_t launch_router_tc(const LayerDev& L, const uint16_t* x, int T, float* logits,
                             uint16_t* hi, uint16_t* lo, bool split, Control* ctl,
                             cudaStream_t st) {
  cudaError_t e = cudaSuccess;
  if (split) {
    e = launch_split_router(L.Wr, L.E, L.d, hi, lo, st);
    if (e != cudaSuccess) return e;
  }
  RtMaps mp;
  if (!make_map_b16(&mp.hi, hi, (uint64_t)L.d, (uint64_t)L.E) ||
      !make_map_b16(&mp.lo, lo, (uint64_t)L.d, (uint64_t)L.E) ||
      !make_map_b16(&mp.x, x, (uint64_t)L.d, (uint64_t)T))
    return cudaErrorInvalidValue;
  const size_t sm = router_tc_smem();
  e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid((L.E + 127) / 128, (T + 127) / 128);
  return launch_pdl(router_tc_kernel, grid, dim3(RT_THREADS), sm, st,
                    static_cast<const float*>(L.bias), L.E, T, L.d, logits, ctl, mp);
}

}  // namespace moe
