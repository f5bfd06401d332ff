// select.cuh -- per-token top-k selection with softmax renormalisation, and
// staging of a token window (optional RMSNorm) into shared memory; used by the
// small-window router (selection in its last CTA) and the batch top-k kernel
// of long windows.
//
// Selection: the router keeps the top_k of the expert scores ("Strata
// open-source runtime", section "the model itself": 10 of 512 per layer);
// largest first, equal logits to the lower expert index, NaN last; the weights
// are the softmax of the selected logits.
#pragma once
#include "common.cuh"
#include "moe.h"

namespace moe {

constexpr float kRmsEps = 1e-6f;

// ---------------------------------------------------------------- selection
// One warp selects top_k of E (E <= 1024) logits of one token and writes the
// ids (largest first) and renormalised weights.  Each lane keeps the best of
// its own logits (ties: lowest index, as the lane scans upward); a round takes
// the warp maximum of the keys and the lowest index holding it (two redux
// instructions), and only the winning lane rescans.  NPER >= E / 32 logits per
// lane.  LEAN picks how a lane rescans: a running comparison (few registers,
// for the batch top-k kernel whose occupancy they limit) or a tree over
// packed (key, ~index) pairs (a shorter dependency chain per round, for the
// latency of one small window).  Both choose the same entry.
template <int NPER, bool PREF, bool LEAN = false>
__device__ void warp_topk_n(const float* __restrict__ row, const float* __restrict__ pref,
                            float* __restrict__ counts, int E, int k, int32_t* __restrict__ ids,
                            float* __restrict__ w, Control* ctl, bool debug) {
  const int lane = threadIdx.x & 31;
  // all loads first (independent, in flight together), checks afterwards
  float v[NPER], b[PREF ? NPER : 1];
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldcg(row + e) : 0.f;
    if (PREF) b[i] = e < E ? __ldg(pref + e) : 0.f;
  }
  // selection key: the logit, plus the expert's selection bonus when given
  // (fp32 add); the weights below use the logits alone
  uint32_t key[NPER];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int e = lane + 32 * i;
    key[i] = order_key(PREF ? v[i] + b[PREF ? i : 0] : v[i]);
    bad |= (e < E) && !isfinite(v[i]);
  }
  if (debug && bad) record_error(ctl, kErrNonFinite, 0x100);
  uint32_t taken = 0;
  // lane-local best: a scan in ascending expert index in which only a
  // strictly larger key replaces the best, so equal keys stay with the lower
  // index (a NaN, key 0, wins only where nothing else is left); bi =
  // 0xFFFFFFFF when every entry of the lane is taken or outside E
  uint32_t bk = 0u, bi = 0xFFFFFFFFu;
  auto rescan = [&]() {
    if constexpr (LEAN) {
      uint32_t k0 = 0u, i0 = 0xFFFFFFFFu;
#pragma unroll
      for (int i = 0; i < NPER; ++i) {
        const uint32_t e = (uint32_t)(lane + 32 * i);
        const bool ok = ((int)e < E) && !((taken >> i) & 1u);
        if (ok && (i0 == 0xFFFFFFFFu || key[i] > k0)) {
          k0 = key[i];
          i0 = e;
        }
      }
      bk = k0;
      bi = i0;
    } else {
      // (key << 32 | ~index): the larger key wins, equal keys go to the lower
      // index; 0 marks an entry that is taken or outside E
      unsigned long long c[NPER];
#pragma unroll
      for (int i = 0; i < NPER; ++i) {
        const uint32_t e = (uint32_t)(lane + 32 * i);
        const bool ok = ((int)e < E) && !((taken >> i) & 1u);
        c[i] = ok ? ((unsigned long long)key[i] << 32) | (unsigned long long)(~e) : 0ull;
      }
#pragma unroll
      for (int half = NPER / 2; half >= 1; half >>= 1) {
#pragma unroll
        for (int i = 0; i < half; ++i) c[i] = c[i + half] > c[i] ? c[i + half] : c[i];
      }
      bk = c[0] ? (uint32_t)(c[0] >> 32) : 0u;
      bi = c[0] ? ~(uint32_t)(c[0] & 0xFFFFFFFFull) : 0xFFFFFFFFu;
    }
  };
  rescan();
  float my_v = 0.f;
  uint32_t my_id = 0;
  for (int j = 0; j < k; ++j) {
    const uint32_t mk = __reduce_max_sync(0xffffffffu, bi == 0xFFFFFFFFu ? 0u : bk);
    const uint32_t win = __reduce_min_sync(0xffffffffu, (bi != 0xFFFFFFFFu && bk == mk) ? bi : 0xFFFFFFFFu);
    const uint32_t u = (mk & 0x80000000u) ? (mk & 0x7FFFFFFFu) : ~mk;
    if (PREF) {   // the unbiased logit of the pick, from the lane that holds it
      float own = 0.f;
#pragma unroll
      for (int i = 0; i < NPER; ++i)
        if ((win >> 5) == (uint32_t)i) own = v[i];
      const float vj = __shfl_sync(0xffffffffu, own, win & 31u);
      if (lane == j) my_v = vj;
    } else if (lane == j) {
      my_v = __uint_as_float(u);
    }
    if (lane == j) my_id = win;
    if (lane == 0) ids[j] = static_cast<int32_t>(win);
    if ((win & 31u) == (uint32_t)lane) {
      taken |= 1u << (win >> 5);
      rescan();
    }
  }
  // softmax reference: the largest selected logit (the first pick without a
  // selection bonus; with one, the picks are re-read unbiased and maximised)
  float v0;
  if (PREF) {
    const uint32_t mk = __reduce_max_sync(0xffffffffu, lane < k ? order_key(my_v) : 0u);
    v0 = __uint_as_float((mk & 0x80000000u) ? (mk & 0x7FFFFFFFu) : ~mk);
  } else {
    v0 = __shfl_sync(0xffffffffu, my_v, 0);
  }
  // routing counters (adaptive slot layout): one count per pick
  if (counts && lane < k) atomicAdd(counts + my_id, 1.f);
  const float ex = lane < k ? expf(my_v - v0) : 0.f;
  const float den = warp_sum(ex);
  if (lane < k) w[lane] = ex / den;
}

// The variants with a selection bonus are kept out of line: their extra
// register arrays then leave the plain path's allocation alone.
template <int NPER, bool LEAN>
__device__ __noinline__ void warp_topk_pref(const float* __restrict__ row,
                                            const float* __restrict__ pref,
                                            float* __restrict__ counts, int E, int k,
                                            int32_t* __restrict__ ids, float* __restrict__ w,
                                            Control* ctl, bool debug) {
  warp_topk_n<NPER, true, LEAN>(row, pref, counts, E, k, ids, w, ctl, debug);
}

template <bool LEAN = false>
__device__ __forceinline__ void warp_topk(const float* __restrict__ row, const float* __restrict__ pref,
                                          float* __restrict__ counts, int E, int k,
                                          int32_t* __restrict__ ids, float* __restrict__ w,
                                          Control* ctl, bool debug) {
  if (pref) {
    if (E <= 128)
      warp_topk_pref<4, LEAN>(row, pref, counts, E, k, ids, w, ctl, debug);
    else if (E <= 512)
      warp_topk_pref<16, LEAN>(row, pref, counts, E, k, ids, w, ctl, debug);
    else
      warp_topk_pref<32, LEAN>(row, pref, counts, E, k, ids, w, ctl, debug);
  } else {
    if (E <= 128)
      warp_topk_n<4, false, LEAN>(row, pref, counts, E, k, ids, w, ctl, debug);
    else if (E <= 512)
      warp_topk_n<16, false, LEAN>(row, pref, counts, E, k, ids, w, ctl, debug);
    else
      warp_topk_n<32, false, LEAN>(row, pref, counts, E, k, ids, w, ctl, debug);
  }
}

// --------------------------------------------------------- x (bf16) staging
// Loads T token rows into shared memory as bf16 bits (16-byte accesses); with
// PRENORM replaces them by bf16(x / sqrt(mean(x^2) + eps)), computed in fp32.
// The sum of squares of a token is taken by one warp in a fixed order, so the
// result does not depend on scheduling.  red: >= T floats.  Ends with a block
// barrier.
__device__ __forceinline__ void stage_tokens(const uint16_t* __restrict__ x, int T, int d,
                                             bool prenorm, uint16_t* xs, float* red) {
  const int tid = threadIdx.x, nt = blockDim.x, warp = tid >> 5, lane = tid & 31;
  if (prenorm) {
    for (int t = warp; t < T; t += nt >> 5) {
      float ss = 0.f;
      for (int i = lane * 8; i < d; i += 256) {
        const uint4 v = *reinterpret_cast<const uint4*>(x + (size_t)t * d + i);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float a = __uint_as_float(w4[j] << 16), b = __uint_as_float(w4[j] & 0xFFFF0000u);
          ss += a * a + b * b;
        }
      }
      ss = warp_sum(ss);
      if (lane == 0) red[t] = rsqrtf(ss / (float)d + kRmsEps);
    }
    __syncthreads();
  }
  const int per = d / 8;
  for (int i = tid; i < T * per; i += nt) {
    uint4 v = reinterpret_cast<const uint4*>(x)[i];
    if (prenorm) {
      const float inv = red[i / per];
      uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(w4[j] << 16) * inv,
                                                       __uint_as_float(w4[j] & 0xFFFF0000u) * inv);
        w4[j] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      v = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    reinterpret_cast<uint4*>(xs)[i] = v;
  }
  __syncthreads();
}

}  // namespace moe
