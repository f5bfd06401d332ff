// prefill.cu -- prefill expert step: bucketing + tcgen05 grouped GEMMs.
//
// A prompt chunk of thousands of tokens routes to nearly every expert of a
// layer, and each expert's weights are then used by the whole chunk ("Why
// Strata is fast on low-VRAM GPUs", section "reading long prompts"): the work
// is a grouped dense contraction, so it runs on the tensor cores.
//
//  1. prep:    x16 = fp16(x or bf16(RMSNorm(x)))                   [T][d]
//  2. bucket:  per-expert counts, exclusive scan, stable scatter of the
//              (token, slot) entries in ascending token order; the shared
//              expert is bucket E with every token; a chunk table splits each
//              bucket into tiles of at most 128 tokens.
//  3. gather:  xperm[position] = x16[token of position] (bucket order).
//  4. GEMM1:   for each (chunk, pair of 64-feature tiles): two D[128 x n] =
//              A . B^T, each A = 64 gate rows and the 64 matching up rows of
//              the expert, dequantised from the packed 2/3-bit codes into a
//              128-byte swizzled fp16 tile by producer warps; B = the chunk's
//              token rows of xperm, loaded once per k-step by TMA and shared by
//              both tiles.  tcgen05.mma accumulates in TMEM; the epilogue reads
//              TMEM, applies SwiGLU and stores the hidden rows H[position][f]
//              (fp16).
//  5. GEMM2:   for each (chunk, pair of 128-row tiles of d): D = Wd_tile .
//              H_chunk^T; the epilogue scales column n by its routing weight
//              and adds it into y_acc[token][i] (fp32 reductions), or, with
//              MOE_F_DETERMINISTIC, stores it as row `position` of ybuf.
//  6. finalize y = bf16(y_acc (+ x)), or the fixed-order sum of the ybuf rows
//              of each token (+ x).
//
// Warp roles of the GEMM kernel (one CTA per SM, persistent over work items):
//  warps 0-3   epilogue (TMEM lane quadrant = warp index)
//  warps 4-11  A producers: each thread dequantises one 32-value group of a row
//              of both A tiles from the packed codes staged in a small ring
//  warp 12     TMEM allocation and the single MMA-issuing thread
//  warp 13     loads: the B tile of every k-step by TMA (rows of the permuted
//              token buffer, or of H), and the packed codes by bulk copies
// Every wait is bounded; a timed-out role records the error and stops waiting.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include "internal.h"
#include "tc.cuh"

namespace moe {

cudaError_t launch_prep_tokens(const uint16_t* x, int T, int d, uint32_t flags, uint16_t* xn,
                               __half* x16, Control* ctl, cudaStream_t st);

constexpr int PF_NT = 128;        // token tile = MMA N (max)
constexpr int PF_BM = 128;        // MMA M
constexpr int PF_NSA = 3;         // A (dequantised weights) ring stages: produced on chip
constexpr int PF_NSB = 4;         // B (token rows) ring stages: loaded from memory by TMA
constexpr int PF_CS = 6;          // packed-code ring stages
constexpr int PF_TOKBLK = 256;    // bucketing token block
// Code stage of one k-step of a tile pair (two groups of 16 packed 16-row
// tiles), as the 4-D tensor-map boxes land: [tile][group][bytes].
//  gate/up: Wg lo [8][2][128] @0 | Wu lo @2048 | Wg hi [8][2][64] @4096 | Wu hi @5120
//           | Wg scales [8][2][32] @6144 | Wu scales @6656
//  down:    Wd lo [16][2][128] @0 | Wd hi [16][2][64] @4096 | Wd scales [16][2][32] @6144
constexpr int PF_CODE_STAGE = 7168;
constexpr int PF_A_TILE = PF_BM * 128;     // one 128 x 64 fp16 tile
constexpr int PF_A_STAGE = 2 * PF_A_TILE;  // a tile pair
constexpr int PF_B_STAGE = PF_NT * 128;
constexpr int PF_THREADS = 14 * 32;
constexpr int PF_A_THREADS = 256;

struct PfWs {
  int* counts;      // [E+1]
  int* misc;        // [16]: misc[0] = number of chunks
  int* offsets;     // [E+2]
  int* entries;     // [T*k]
  int* blockcnt;    // [nblk][E]
  int4* chunks;     // [maxC]
  int* tokpos;      // [T*(k+1)]
  float* wpos;      // [T*(k+1)]
  __half* H;        // [(T*(k+1) + 128)][Fmax]
  float* yacc;      // [T][d]
  __half* x16;      // [T][d]
  uint16_t* xn;     // [T][d]
  int* invpos;      // [T*k]: position of entry t*k+j in the buckets (-1: invalid id)
  __half* xperm;    // [T*(k+1)][d]: token rows in bucket order (GEMM1 operand)
  float* ybuf;      // [T*(k+1)][d]: weighted expert rows (deterministic GEMM2), aliases xperm
};

static size_t pf_max_chunks(const LayerDev& L, int T) {
  return (size_t)T * L.k / PF_NT + L.E + (T + PF_NT - 1) / PF_NT + 2;
}

size_t prefill_ws_bytes(const LayerDev& L, int T, size_t* parts) {
  const int Fmax = L.F > L.Fs ? L.F : L.Fs;
  const size_t nblk = ((size_t)T + PF_TOKBLK - 1) / PF_TOKBLK;
  const size_t R = (size_t)T * (L.k + 1);
  parts[0] = (size_t)T * L.d * 2;                              // xn
  parts[1] = (size_t)T * L.d * 2;                              // x16
  parts[2] = (size_t)(L.E + 1 + 16) * 4;                       // counts + misc
  parts[3] = (size_t)(L.E + 2) * 4;                            // offsets
  parts[4] = (size_t)T * L.k * 4;                              // entries
  parts[5] = nblk * L.E * 4;                                   // blockcnt
  parts[6] = pf_max_chunks(L, T) * 16 + 256 + 2 * (R * 4 + 256) + (size_t)T * L.k * 4;
                                                               // chunks, tokpos, wpos, invpos
  parts[7] = (R + PF_NT) * Fmax * 2;                           // H
  parts[8] = (size_t)T * L.d * 4;                              // yacc
  parts[9] = R * L.d * 4;                                      // xperm / ybuf
  size_t tot = 0;
  for (int i = 0; i < 10; ++i) tot += parts[i];
  return tot;
}

static PfWs pf_ws(const LayerDev& L, int T, char* ws, const WsLayout& lay) {
  PfWs p;
  p.xn = reinterpret_cast<uint16_t*>(ws + lay.xn);
  p.x16 = reinterpret_cast<__half*>(ws + lay.x16);
  p.counts = reinterpret_cast<int*>(ws + lay.counts);
  p.misc = p.counts + L.E + 1;
  p.offsets = reinterpret_cast<int*>(ws + lay.offsets);
  p.entries = reinterpret_cast<int*>(ws + lay.entries);
  p.blockcnt = reinterpret_cast<int*>(ws + lay.blockcnt);
  char* t = ws + lay.tiles;
  p.chunks = reinterpret_cast<int4*>(t);
  t += (pf_max_chunks(L, T) * 16 + 255) / 256 * 256;
  p.tokpos = reinterpret_cast<int*>(t);
  const size_t R = (size_t)T * (L.k + 1);
  t += (R * 4 + 255) / 256 * 256;
  p.wpos = reinterpret_cast<float*>(t);
  t += (R * 4 + 255) / 256 * 256;
  p.invpos = reinterpret_cast<int*>(t);
  p.H = reinterpret_cast<__half*>(ws + lay.h);
  p.yacc = reinterpret_cast<float*>(ws + lay.yacc);
  p.xperm = reinterpret_cast<__half*>(ws + lay.xperm);
  p.ybuf = reinterpret_cast<float*>(ws + lay.xperm);
  return p;
}

// ---------------------------------------------------------------- bucketing
__global__ void __launch_bounds__(256) bucket_hist_kernel(const int32_t* __restrict__ ids, int T,
                                                          int k, int E, int* __restrict__ blockcnt,
                                                          Control* ctl) {
  extern __shared__ int hist[];
  pdl_wait();
  pdl_launch_dependents();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * PF_TOKBLK, t1 = min(T, t0 + PF_TOKBLK);
  for (int i = t0 * k + threadIdx.x; i < t1 * k; i += blockDim.x) {
    const int e = ids[i];
    if (e >= 0 && e < E)
      atomicAdd(&hist[e], 1);
    else
      record_error(ctl, kErrRange, 0x600);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) blockcnt[(size_t)blockIdx.x * E + e] = hist[e];
}

// In-place exclusive scan of v[0..n) (n <= 2048) by a 1024-thread block;
// returns the total.
__device__ int block_excl_scan(int* v, int n, int* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i0 = 2 * tid, i1 = 2 * tid + 1;
  const int a = i0 < n ? v[i0] : 0, b = i1 < n ? v[i1] : 0;
  int s = a + b, inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int wv = warp_tot[lane], wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_tot[lane] = wi - wv;   // exclusive prefix of warp totals
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  const int excl = warp_tot[warp] + inc - s;
  if (i0 < n) v[i0] = excl;
  if (i1 < n) v[i1] = excl + a;
  const int total = warp_tot[32];
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(1024) bucket_scan_kernel(int* __restrict__ blockcnt, int nblk,
                                                           int E, int T, int k, int has_shared,
                                                           const int32_t* __restrict__ slot, PfWs p,
                                                           int* __restrict__ user_offsets,
                                                           Control* ctl) {
  __shared__ int cnt[2048], off[2048], nch[2048], wt[33];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
    for (int b = 0; b < nblk; ++b) {
      const int c = blockcnt[(size_t)b * E + e];
      blockcnt[(size_t)b * E + e] = run;
      run += c;
    }
    cnt[e] = run;
  }
  if (tid == 0) cnt[E] = has_shared ? T : 0;   // the shared expert: every token
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) {
    off[e] = cnt[e];
    nch[e] = (cnt[e] + PF_NT - 1) / PF_NT;
  }
  __syncthreads();
  block_excl_scan(off, E + 1, wt);
  const int nchunks = block_excl_scan(nch, E + 1, wt);
  for (int e = tid; e <= E; e += blockDim.x) {
    p.counts[e] = cnt[e];
    p.offsets[e] = off[e];
    if (user_offsets) user_offsets[e] = off[e];
    // chunk record: (bucket, first position, rows, weight slot of the bucket)
    int s = 0;
    if (e < E && cnt[e] > 0) {
      s = slot[e];
      if (s < 0 || s >= E) {
        record_error(ctl, kErrRange, 0x601);
        s = 0;
      }
    }
    for (int c = 0; c * PF_NT < cnt[e]; ++c)
      p.chunks[nch[e] + c] = make_int4(e, off[e] + c * PF_NT, min(PF_NT, cnt[e] - c * PF_NT), s);
  }
  if (tid == 0) {
    p.offsets[E + 1] = off[E] + cnt[E];
    p.misc[0] = nchunks;
  }
}

__global__ void __launch_bounds__(256) bucket_scatter_kernel(const int32_t* __restrict__ ids,
                                                             const float* __restrict__ w, int T,
                                                             int k, int E, int has_shared, PfWs p,
                                                             int32_t* __restrict__ user_entries) {
  extern __shared__ uint32_t bits[];   // [E][8]: token bitmap of this block per expert
  pdl_wait();
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < E * 8; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  const int t0 = blockIdx.x * PF_TOKBLK, t1 = min(T, t0 + PF_TOKBLK);
  for (int i = t0 * k + threadIdx.x; i < t1 * k; i += blockDim.x) {
    const int e = ids[i], lt = i / k - t0;
    if (e >= 0 && e < E) atomicOr(&bits[e * 8 + (lt >> 5)], 1u << (lt & 31));
  }
  __syncthreads();
  for (int i = t0 * k + threadIdx.x; i < t1 * k; i += blockDim.x) {
    const int e = ids[i], t = i / k, lt = t - t0;
    if (e < 0 || e >= E) {
      p.invpos[i] = -1;
      continue;
    }
    int rank = __popc(bits[e * 8 + (lt >> 5)] & ((1u << (lt & 31)) - 1u));
    for (int wd = 0; wd < (lt >> 5); ++wd) rank += __popc(bits[e * 8 + wd]);
    const int pos = p.offsets[e] + p.blockcnt[(size_t)blockIdx.x * E + e] + rank;
    p.entries[pos] = i;
    p.invpos[i] = pos;
    if (user_entries) user_entries[pos] = i;
    p.tokpos[pos] = t;
    p.wpos[pos] = w[i];
  }
  if (has_shared) {
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
      const int pos = p.offsets[E] + t;   // the shared bucket follows the routed ones
      p.tokpos[pos] = t;
      p.wpos[pos] = 1.f;
    }
  }
}

// Token rows in bucket order: xperm[pos] = x16[tokpos[pos]] for the filled
// positions pos < offsets[E+1] (routed buckets, then the shared bucket).
__global__ void __launch_bounds__(256) gather_rows_kernel(const __half* __restrict__ x16,
                                                          const int* __restrict__ tokpos,
                                                          const int* __restrict__ offsets, int E,
                                                          int T, __half* __restrict__ xperm,
                                                          int d, Control* ctl) {
  pdl_wait();
  pdl_launch_dependents();
  const int per = d / 8;
  const long long n = (long long)offsets[E + 1] * per;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long pos = i / per;
    const int c = (int)(i - pos * per);
    int t = tokpos[pos];
    if (t < 0 || t >= T) {
      record_error(ctl, kErrRange, 0x602);
      t = 0;
    }
    reinterpret_cast<uint4*>(xperm)[i] = reinterpret_cast<const uint4*>(x16 + (size_t)t * d)[c];
  }
}

// ----------------------------------------------------------------- GEMM
struct PfArgs {
  LayerDev L;
  int mode;     // 0: gate/up -> H,  1: down -> y_acc (or ybuf)
  int T;
  int Fmax;
  int ppc;      // tile pairs (work items) per chunk
  int det;      // mode 1: store each position's row to ybuf instead of reducing
  PfWs p;
  Control* ctl;
};

// Work item = (chunk, tile pair).  A tile pair is two 128-row A tiles that
// share every B tile: gate/up rows of 2 x 64 features (mode 0) or 2 x 128 rows
// of the down projection (mode 1).
struct PfItem {
  int u, pos0, nv, pair, slot, F, KS, ng_last;
  bool shared, two, valid;
};

__device__ __forceinline__ PfItem pf_item(const PfArgs& a, int4 ch, int pair) {
  PfItem it;
  it.u = ch.x;
  it.pos0 = ch.y;
  it.nv = ch.z;
  it.slot = ch.w;
  it.pair = pair;
  it.shared = it.u >= a.L.E;
  it.F = it.shared ? a.L.Fs : a.L.F;
  const int K = a.mode == 0 ? a.L.d : it.F;
  it.KS = (K + 63) / 64;
  it.ng_last = K / kGroup - 2 * (it.KS - 1);
  if (a.mode == 0) {
    it.valid = it.nv > 0 && pair * 128 < it.F;
    it.two = (2 * pair + 1) * 64 < it.F;
  } else {
    it.valid = it.nv > 0 && it.F > 0 && pair * 2 * PF_BM < a.L.d;
    it.two = (2 * pair + 1) * PF_BM < a.L.d;
  }
  return it;
}

// This CTA's work items in order (i = blockIdx.x + j * gridDim.x), skipping
// empty ones; the chunk record of the next item is loaded one item ahead.
struct ItemSeq {
  int i, n, ppc;
  int4 next;
  __device__ __forceinline__ void init(const PfArgs& a, int n_items) {
    i = blockIdx.x;
    n = n_items;
    ppc = a.ppc;
    next = make_int4(0, 0, 0, 0);
    if (i < n) next = __ldg(a.p.chunks + i / ppc);
  }
  __device__ __forceinline__ bool get(const PfArgs& a, PfItem& it) {
    for (;;) {
      if (i >= n) return false;
      const int4 ch = next;
      const int pair = i % ppc;
      i += gridDim.x;
      if (i < n) next = __ldg(a.p.chunks + i / ppc);
      it = pf_item(a, ch, pair);
      if (it.valid) return true;
    }
  }
};

// (item, k-step) sequence, in the order every role walks it.
struct KSeq {
  ItemSeq s;
  PfItem it;
  int ks;
  bool done;
  __device__ __forceinline__ const PfItem& item_ref() const { return it; }
  __device__ __forceinline__ void init(const PfArgs& a, int n_items) {
    s.init(a, n_items);
    done = !s.get(a, it);
    ks = 0;
  }
  __device__ __forceinline__ void advance(const PfArgs& a) {
    if (++ks >= it.KS) {
      done = !s.get(a, it);
      ks = 0;
    }
  }
};

// Tensor maps: the token (or hidden) rows of the B operand, and the packed
// codes / scales of the routed experts and of the shared expert viewed as
// 4-D byte tensors [bytes of a group][group][16-row tile][slot].
struct alignas(64) PfMaps {
  CUtensorMap b;
  CUtensorMap lo, hi, sc;      // routed experts
  CUtensorMap slo, shi, ssc;   // shared expert
};

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// One lane: the packed codes and scales of k-step ks of `it` (both tiles of
// the pair) into a code stage; the layout is given at PF_CODE_STAGE.
template <int BITS>
__device__ __forceinline__ void pf_issue_codes(const PfArgs& a, const PfMaps& mp, const PfItem& it,
                                               int ks, unsigned char* st, uint64_t* bar) {
  const CUtensorMap* lo = it.shared ? &mp.slo : &mp.lo;
  const CUtensorMap* hi = it.shared ? &mp.shi : &mp.hi;
  const CUtensorMap* sc = it.shared ? &mp.ssc : &mp.sc;
  const int g0 = 2 * ks;
  mbar_arrive_expect_tx(bar, 5120 + (BITS == 3 ? 2048 : 0));
  if (a.mode == 0) {
    const int tg = 8 * it.pair, tu = it.F / kTileRows + 8 * it.pair;
    tma_load_4d(st, lo, 0, g0, tg, it.slot, bar);
    tma_load_4d(st + 2048, lo, 0, g0, tu, it.slot, bar);
    if (BITS == 3) {
      tma_load_4d(st + 4096, hi, 0, g0, tg, it.slot, bar);
      tma_load_4d(st + 5120, hi, 0, g0, tu, it.slot, bar);
    }
    tma_load_4d(st + 6144, sc, 0, g0, tg, it.slot, bar);
    tma_load_4d(st + 6656, sc, 0, g0, tu, it.slot, bar);
  } else {
    const int t0 = 16 * it.pair;
    tma_load_4d(st, lo, 0, g0, t0, it.slot, bar);
    if (BITS == 3) tma_load_4d(st + 4096, hi, 0, g0, t0, it.slot, bar);
    tma_load_4d(st + 6144, sc, 0, g0, t0, it.slot, bar);
  }
}

// Dequantise chunk m (8 consecutive K values) of one group into fp16.  The
// code q of a value sits in a half's mantissa under the exponent of 1024
// (magic 0x6400), scaled by 4^-m for its bit position; one fma recentres it
// to q - 2^(b-1) exactly, and the multiply by the fp16 scale is the only
// rounding step.
template <int BITS>
__device__ __forceinline__ uint4 pf_dq_chunk(const uint32_t (&X)[4], const uint32_t (&Y)[4], int m,
                                             __half2 s2) {
  const uint32_t magic = 0x64006400u;
  const uint32_t mask = 0x00030003u << (2 * m);
  const float mulR = m == 0 ? 1.f : (m == 1 ? 0.25f : (m == 2 ? 0.0625f : 0.015625f));
  uint32_t out[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const __half2 R = u32_as_h2(and_or(X[t], mask, magic));
    __half2 v;
    if (BITS == 2) {
      const float addR = m == 0 ? -1026.f : (m == 1 ? -258.f : (m == 2 ? -66.f : -18.f));
      v = __hfma2(R, __float2half2_rn(mulR), __float2half2_rn(addR));
    } else {
      const float mulH = m == 0 ? 4.f : (m == 1 ? 2.f : (m == 2 ? 1.f : 0.5f));
      const float addH = m == 0 ? -5124.f : (m == 1 ? -2308.f : (m == 2 ? -1092.f : -532.f));
      const __half2 H = u32_as_h2(and_or(Y[t], 0x00010001u << m, magic));
      const __half2 tmp = __hfma2(H, __float2half2_rn(mulH), __float2half2_rn(addH));
      v = __hfma2(R, __float2half2_rn(mulR), tmp);
    }
    out[t] = h2_as_u32(__hmul2(v, s2));
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// One (row, group) unit of an A tile: read its codes and scale from the code
// stage (zeros when the row or group is outside the matrix).
template <int BITS>
__device__ __forceinline__ void pf_read_unit(const unsigned char* cst, bool use, int lo_off,
                                             int hi_off, int sc_off, uint32_t (&X)[4],
                                             uint32_t (&Y)[4], __half2& s2) {
  if (use) {
    const uint2 lo = *reinterpret_cast<const uint2*>(cst + lo_off);
    const uint32_t hi = BITS == 3 ? *reinterpret_cast<const uint32_t*>(cst + hi_off) : 0u;
    s2 = __half2half2(*reinterpret_cast<const __half*>(cst + sc_off));
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      X[t] = __byte_perm(lo.x, lo.y, (uint32_t)t | ((uint32_t)(4 + t) << 8));
      Y[t] = hi >> (4 * t);
    }
  } else {
    s2 = __float2half2_rn(0.f);
#pragma unroll
    for (int t = 0; t < 4; ++t) X[t] = Y[t] = 0u;
  }
}

struct PfSmem {
  size_t a, b, codes, stage_h, bars, holder, total;
};
__host__ __device__ inline PfSmem pf_smem() {
  PfSmem m;
  size_t o = 0;
  m.a = o;
  o += (size_t)PF_NSA * PF_A_STAGE;
  m.b = o;
  o += (size_t)PF_NSB * PF_B_STAGE;
  m.codes = o;
  o += (size_t)PF_CS * PF_CODE_STAGE;
  m.stage_h = o;                       // epilogue staging of H rows: [128 n][64 f] fp16
  o += (size_t)PF_NT * 64 * 2;
  m.bars = o;
  o += (2 * PF_NSA + 2 * PF_NSB + 2 * PF_CS + 4) * 8;
  m.holder = o;
  o += 16;
  m.total = o + 1024;   // slack to align the base to 1024
  return m;
}

template <int BITS>
__global__ void __launch_bounds__(PF_THREADS, 1) pf_gemm_kernel(const PfArgs a,
                                                                 const __grid_constant__ PfMaps mp) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const PfSmem m = pf_smem();
  unsigned char* sA = smem + m.a;
  unsigned char* sB = smem + m.b;
  unsigned char* sC = smem + m.codes;
  __half* sH = reinterpret_cast<__half*>(smem + m.stage_h);
  uint64_t* fullA = reinterpret_cast<uint64_t*>(smem + m.bars);
  uint64_t* emptyA = fullA + PF_NSA;
  uint64_t* fullB = emptyA + PF_NSA;
  uint64_t* emptyB = fullB + PF_NSB;
  uint64_t* cfull = emptyB + PF_NSB;
  uint64_t* cempty = cfull + PF_CS;
  uint64_t* tfull = cempty + PF_CS;
  uint64_t* tempty = tfull + 2;
  uint32_t* holder = reinterpret_cast<uint32_t*>(smem + m.holder);
  Control* ctl = a.ctl;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < PF_NSA; ++s) {
      mbar_init(&fullA[s], PF_A_THREADS);
      mbar_init(&emptyA[s], 1);
    }
    for (int s = 0; s < PF_NSB; ++s) {
      mbar_init(&fullB[s], 1);
      mbar_init(&emptyB[s], 1);
    }
    for (int c = 0; c < PF_CS; ++c) {
      mbar_init(&cfull[c], 1);
      mbar_init(&cempty[c], PF_A_THREADS);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
    }
    fence_barrier_init();
  }
  if (warp == 12) {
    tmem_alloc(holder, 512);
    tmem_relinquish();
  }
  if (warp == 13 && lane < 7) {   // the seven tensor-map descriptors into the TMA unit's cache
    const CUtensorMap* maps[7] = {&mp.b, &mp.lo, &mp.hi, &mp.sc, &mp.slo, &mp.shi, &mp.ssc};
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(maps[lane])) : "memory");
  }
  pdl_wait();
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *holder;
  const int n_items = a.p.misc[0] * a.ppc;
  bool ok = true;

  if (warp >= 4 && warp < 12) {
    // ------------------------------------------------ A producers (dequant)
    // Thread = (row r of both tiles, group gi of the k-step).
    const int ta = tid - 128;
    const int r = ta >> 1, gi = ta & 1, rr = r & 15;
    int lo_off, hi_off, sc_off, dlo, dhi, dsc, blk0, dblk;
    if (a.mode == 0) {
      // rows of a tile: four blocks of [16 gate rows, 16 up rows]
      const int qt = r >> 5, isu = (r >> 4) & 1;
      lo_off = isu * 2048 + qt * 256;
      hi_off = 4096 + isu * 1024 + qt * 128;
      sc_off = 6144 + isu * 512 + qt * 64;
      dlo = 1024, dhi = 512, dsc = 256;
      blk0 = qt, dblk = 4;   // 16-row feature block within the pair
    } else {
      const int q16 = r >> 4;
      lo_off = q16 * 256;
      hi_off = 4096 + q16 * 128;
      sc_off = 6144 + q16 * 64;
      dlo = 2048, dhi = 1024, dsc = 512;
      blk0 = q16, dblk = 8;
    }
    lo_off += gi * 128 + rr * 8;
    hi_off += gi * 64 + rr * 4;
    sc_off += gi * 32 + rr * 2;
    const int nblk = a.mode == 0 ? 0 : a.L.d / kTileRows;   // mode 0: set per item
    unsigned char* const adst = sA + r * 128;
    KSeq cur;
    cur.init(a, n_items);
    int cs = 0, sa = 0;
    uint32_t pc = 0, pa = 0;
    int g = 0;
    while (!cur.done) {
      const PfItem& it = cur.item_ref();
      const int ng = cur.ks == it.KS - 1 ? it.ng_last : 2;
      const int rows_blk = a.mode == 0 ? it.F / kTileRows : nblk;
      const int b0 = (a.mode == 0 ? 8 : 16) * it.pair + blk0;
      const bool u0 = gi < ng && b0 < rows_blk;
      const bool u1 = gi < ng && b0 + dblk < rows_blk && it.two;
      if (ok) ok = mbar_wait(&cfull[cs], pc, ctl, 0x610);
      uint32_t X0[4], Y0[4], X1[4], Y1[4];
      __half2 s0, s1;
      const unsigned char* cst = sC + cs * PF_CODE_STAGE;
      pf_read_unit<BITS>(cst, u0 && ok, lo_off, hi_off, sc_off, X0, Y0, s0);
      pf_read_unit<BITS>(cst, u1 && ok, lo_off + dlo, hi_off + dhi, sc_off + dsc, X1, Y1, s1);
      mbar_arrive(&cempty[cs]);   // code stage read
      if (++cs == PF_CS) {
        cs = 0;
        pc ^= 1u;
      }
      uint4 c0[4], c1[4];
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) c0[mm] = pf_dq_chunk<BITS>(X0, Y0, mm, s0);
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) c1[mm] = pf_dq_chunk<BITS>(X1, Y1, mm, s1);
      if (g >= PF_NSA && ok) ok = mbar_wait(&emptyA[sa], pa ^ 1u, ctl, 0x611);
      if (gi < ng) {
        unsigned char* at = adst + sa * PF_A_STAGE;
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
          const int c = 4 * gi + mm;
          *reinterpret_cast<uint4*>(at + ((c ^ (r & 7)) << 4)) = c0[mm];
          *reinterpret_cast<uint4*>(at + PF_A_TILE + ((c ^ (r & 7)) << 4)) = c1[mm];
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&fullA[sa]);
      if (++sa == PF_NSA) {
        sa = 0;
        pa ^= 1u;
      }
      ++g;
      cur.advance(a);
    }
  } else if (warp == 13) {
    // ------------------------------------------------ loads (TMA)
    if (lane == 0) {
      KSeq cur, ahead;
      cur.init(a, n_items);
      ahead.init(a, n_items);
      int g = 0, gc = 0, sb = 0, cs = 0;
      uint32_t pb = 0, pc = 0;
      while (!cur.done) {
        // packed codes up to PF_CS k-steps ahead of the B loads
        while (!ahead.done && gc < g + PF_CS) {
          if (gc >= PF_CS && ok) ok = mbar_wait(&cempty[cs], pc ^ 1u, ctl, 0x621);
          pf_issue_codes<BITS>(a, mp, ahead.item_ref(), ahead.ks, sC + cs * PF_CODE_STAGE, &cfull[cs]);
          if (++cs == PF_CS) {
            cs = 0;
            pc ^= 1u;
          }
          ahead.advance(a);
          ++gc;
        }
        if (g >= PF_NSB && ok) ok = mbar_wait(&emptyB[sb], pb ^ 1u, ctl, 0x620);
        mbar_arrive_expect_tx(&fullB[sb], PF_B_STAGE);
        tma_load_2d(sB + sb * PF_B_STAGE, &mp.b, 64 * cur.ks, cur.item_ref().pos0, &fullB[sb]);
        if (++sb == PF_NSB) {
          sb = 0;
          pb ^= 1u;
        }
        cur.advance(a);
        ++g;
      }
    }
  } else if (warp == 12) {
    // ------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      const uint64_t adesc0 = sw128_kmajor_desc(smem_u32(sA));
      const uint64_t bdesc0 = sw128_kmajor_desc(smem_u32(sB));
      ItemSeq seq;
      seq.init(a, n_items);
      PfItem it;
      int sa = 0, sb = 0, la = 0;
      uint32_t pa = 0, pb = 0;
      while (seq.get(a, it)) {
        const int acc = la & 1;
        if (la >= 2 && ok) ok = mbar_wait(&tempty[acc], ((la >> 1) - 1) & 1, ctl, 0x630);
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(PF_BM, (it.nv + 15) & ~15);
        const uint32_t d0 = tmem_base + (uint32_t)(acc * 256), d1 = d0 + 128;
        const bool two = it.two;
        for (int ks = 0; ks < it.KS; ++ks) {
          if (ok) ok = mbar_wait(&fullB[sb], pb, ctl, 0x632);
          if (ok) ok = mbar_wait(&fullA[sa], pa, ctl, 0x631);
          tc_fence_after();
          const uint64_t ad = adesc0 + (uint64_t)(sa * (PF_A_STAGE >> 4));
          const uint64_t bd = bdesc0 + (uint64_t)(sb * (PF_B_STAGE >> 4));
          const uint32_t first = ks > 0 ? 1u : 0u;
          if (ok) {
            tc_mma_f16(d0, ad, bd, idesc, first);
            tc_mma_f16(d0, ad + 2, bd + 2, idesc, 1u);
            if (two) {
              tc_mma_f16(d1, ad + (PF_A_TILE >> 4), bd, idesc, first);
              tc_mma_f16(d1, ad + (PF_A_TILE >> 4) + 2, bd + 2, idesc, 1u);
            }
            if (ks < it.KS - 1 || it.ng_last == 2) {
              tc_mma_f16(d0, ad + 4, bd + 4, idesc, 1u);
              tc_mma_f16(d0, ad + 6, bd + 6, idesc, 1u);
              if (two) {
                tc_mma_f16(d1, ad + (PF_A_TILE >> 4) + 4, bd + 4, idesc, 1u);
                tc_mma_f16(d1, ad + (PF_A_TILE >> 4) + 6, bd + 6, idesc, 1u);
              }
            }
          }
          tc_commit(&emptyA[sa]);
          tc_commit(&emptyB[sb]);
          if (++sa == PF_NSA) {
            sa = 0;
            pa ^= 1u;
          }
          if (++sb == PF_NSB) {
            sb = 0;
            pb ^= 1u;
          }
        }
        tc_commit(&tfull[acc]);
        ++la;
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 0-3)
    const int q = warp;
    ItemSeq seq;
    seq.init(a, n_items);
    PfItem it;
    int la = 0;
    while (seq.get(a, it)) {
      const int acc = la & 1;
      if (ok) ok = mbar_wait(&tfull[acc], (la >> 1) & 1, ctl, 0x640);
      tc_fence_after();
      const int n_mma = (it.nv + 15) & ~15;
      const int ntile = it.two ? 2 : 1;
      if (a.mode == 0) {
        // SwiGLU into the staging tile sH[n][64 f], then coalesced row stores.
        // TMEM lane 32q + l holds gate row 16q + l (l < 16) or the matching
        // up row (l >= 16); each step pairs two token columns so that every
        // lane computes one output.
        const int fl = 16 * q + (lane & 15);
        const int hi = lane >> 4;
        for (int v = 0; v < ntile; ++v) {
          const uint32_t taddr =
              tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * 256 + v * 128);
          for (int c0 = 0; c0 < n_mma; c0 += 32) {
            uint32_t rv[32];
            tmem_ld_32x32b_x32(taddr + c0, rv);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float a0 = __uint_as_float(rv[j]), a1 = __uint_as_float(rv[j + 1]);
              const float got = __shfl_xor_sync(0xffffffffu, hi ? a0 : a1, 16);
              const float gv = hi ? got : a0;
              const float up = hi ? a1 : got;
              const float h = __fdividef(gv * up, 1.f + __expf(-gv));
              sH[(c0 + j + hi) * 64 + fl] = __float2half_rn(h);
            }
          }
          if (v == ntile - 1) {
            tc_fence_before();
            mbar_arrive(&tempty[acc]);   // TMEM free: the MMA may start item + 2
          }
          named_bar_sync(3, 128);
          const int fcol = 64 * (2 * it.pair + v) + 2 * lane;
          if (ok && fcol < it.F) {
            __half* dst = a.p.H + (size_t)it.pos0 * a.Fmax + fcol;
            for (int n = q; n < it.nv; n += 4)
              *reinterpret_cast<uint32_t*>(dst + (size_t)n * a.Fmax) =
                  *reinterpret_cast<const uint32_t*>(sH + n * 64 + 2 * lane);
          }
          named_bar_sync(3, 128);
        }
      } else {
        for (int v = 0; v < ntile; ++v) {
          const uint32_t taddr =
              tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * 256 + v * 128);
          const int i_out = PF_BM * (2 * it.pair + v) + 32 * q + lane;
          const bool wr = i_out < a.L.d && ok;
          for (int c0 = 0; c0 < n_mma; c0 += 32) {
            uint32_t rv[32];
            tmem_ld_32x32b_x32(taddr + c0, rv);
            // routing weight and destination of column c0 + lane
            const int nl = c0 + lane;
            int tok = 0;
            float wv = 0.f;
            if (nl < it.nv) {
              tok = a.p.tokpos[it.pos0 + nl];
              wv = a.p.wpos[it.pos0 + nl];
            }
            tmem_ld_wait();
            const int jn = min(32, it.nv - c0);
            if (a.det) {
              float* dst = a.p.ybuf + (size_t)(it.pos0 + c0) * a.L.d + i_out;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float wj = __shfl_sync(0xffffffffu, wv, j);
                if (j < jn && wr) dst[(size_t)j * a.L.d] = __uint_as_float(rv[j]) * wj;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float wj = __shfl_sync(0xffffffffu, wv, j);
                const int tj = __shfl_sync(0xffffffffu, tok, j);
                if (j < jn && wr) atomicAdd(a.p.yacc + (size_t)tj * a.L.d + i_out, __uint_as_float(rv[j]) * wj);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
      }
      ++la;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 12) tmem_dealloc(tmem_base, 512);
}

// y = bf16(y_acc (+ x)), four elements per thread.
__global__ void __launch_bounds__(256) prefill_finalize_kernel(const float* __restrict__ yacc,
                                                               const uint16_t* __restrict__ x,
                                                               long long n4, uint32_t flags,
                                                               uint16_t* __restrict__ y) {
  pdl_wait();
  pdl_launch_dependents();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    float4 v = reinterpret_cast<const float4*>(yacc)[i];
    if (flags & MOE_F_RESIDUAL) {
      const uint2 xv = reinterpret_cast<const uint2*>(x)[i];
      v.x += __uint_as_float(xv.x << 16);
      v.y += __uint_as_float(xv.x & 0xFFFF0000u);
      v.z += __uint_as_float(xv.y << 16);
      v.w += __uint_as_float(xv.y & 0xFFFF0000u);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&lo);
    o.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(y)[i] = o;
  }
}

// Fixed-order combine (MOE_F_DETERMINISTIC): y[t] = bf16(sum over j = 0..k-1 of
// ybuf[invpos[t][j]] + ybuf[shared row of t] (+ x[t])), the routed terms in
// selection order and the shared expert last; every term already carries its
// routing weight.
__global__ void __launch_bounds__(256) prefill_finalize_det_kernel(
    const float* __restrict__ ybuf, const int* __restrict__ invpos, const int* __restrict__ offsets,
    const uint16_t* __restrict__ x, int T, int d, int k, int E, int has_shared, uint32_t flags,
    uint16_t* __restrict__ y) {
  pdl_wait();
  pdl_launch_dependents();
  const int per = d / 4;
  const long long n4 = (long long)T * per;
  const int sh0 = offsets[E];
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per), c = (int)(i - (long long)t * per);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int pos = invpos[(size_t)t * k + j];
      if (pos < 0) continue;
      const float4 u = reinterpret_cast<const float4*>(ybuf + (size_t)pos * d)[c];
      v.x += u.x;
      v.y += u.y;
      v.z += u.z;
      v.w += u.w;
    }
    if (has_shared) {
      const float4 u = reinterpret_cast<const float4*>(ybuf + (size_t)(sh0 + t) * d)[c];
      v.x += u.x;
      v.y += u.y;
      v.z += u.z;
      v.w += u.w;
    }
    if (flags & MOE_F_RESIDUAL) {
      const uint2 xv = reinterpret_cast<const uint2*>(x)[i];
      v.x += __uint_as_float(xv.x << 16);
      v.y += __uint_as_float(xv.x & 0xFFFF0000u);
      v.z += __uint_as_float(xv.y << 16);
      v.w += __uint_as_float(xv.y & 0xFFFF0000u);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&lo);
    o.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(y)[i] = o;
  }
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D fp16 row-major tensor [rows][inner] for tiles of PF_NT rows x 64
// elements, 128-byte swizzle (the canonical K-major UMMA layout).
static bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, PF_NT};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D byte tensor [inner bytes][groups][tiles][slots] with the given strides.
static bool make_map4(CUtensorMap* m, const void* base, uint64_t inner, uint64_t groups,
                      uint64_t tiles, uint64_t slots, uint64_t s_group, uint64_t s_tile,
                      uint64_t s_slot, uint32_t box_tiles) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {inner, groups, tiles, slots};
  cuuint64_t strides[3] = {s_group, s_tile, s_slot};
  cuuint32_t box[4] = {(cuuint32_t)inner, 2, box_tiles, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Maps of one expert set (routed: E slots, or the shared expert: 1 slot).
// Boxes cover a tile pair: 8 16-row tiles of Wg (and of Wu) in mode 0, 16
// 16-row tiles of Wd in mode 1.
static bool make_code_maps(const LayerDev& L, int mode, const uint8_t* codes, const uint16_t* scales,
                           int F, uint64_t slots, CUtensorMap* lo, CUtensorMap* hi, CUtensorMap* sc) {
  const int gb = group_bytes(L.bits);
  const uint64_t cbe = 3ull * F * L.d / kGroup * gb, nse2 = 3ull * F * L.d / kGroup * 2;
  const uint64_t nG = L.d / kGroup, nGF = F / kGroup;
  const uint64_t tcb = nG * kTileRows * gb, tcbD = nGF * kTileRows * gb;
  const uint64_t mcb = (uint64_t)(F / kTileRows) * tcb;
  const uint64_t sslot = cbe, sslot_s = nse2;   // slot strides (unused when slots == 1)
  if (mode == 0) {
    const uint64_t tiles = 2ull * F / kTileRows;
    return make_map4(lo, codes, 128, nG, tiles, slots, 128, tcb, sslot, 8) &&
           (L.bits == 2 || make_map4(hi, codes + nG * 128, 64, nG, tiles, slots, 64, tcb, sslot, 8)) &&
           make_map4(sc, scales, 32, nG, tiles, slots, 32, 32 * nG, sslot_s, 8);
  }
  const uint64_t tiles = (uint64_t)L.d / kTileRows;
  const uint8_t* wd = codes + 2 * mcb;
  const uint8_t* wds = reinterpret_cast<const uint8_t*>(scales) + 2ull * F * nG * 2;
  return make_map4(lo, wd, 128, nGF, tiles, slots, 128, tcbD, sslot, 16) &&
         (L.bits == 2 || make_map4(hi, wd + nGF * 128, 64, nGF, tiles, slots, 64, tcbD, sslot, 16)) &&
         make_map4(sc, wds, 32, nGF, tiles, slots, 32, 32 * nGF, sslot_s, 16);
}

template <int BITS>
static cudaError_t launch_gemm(const PfArgs& a, const PfMaps& tm, cudaStream_t st) {
  const PfSmem m = pf_smem();
  cudaError_t e = cudaFuncSetAttribute(pf_gemm_kernel<BITS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)m.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(pf_gemm_kernel<BITS>, dim3(sm_count()), dim3(PF_THREADS), m.total, st, a, tm);
}

cudaError_t launch_prefill(const LayerDev& L, const uint16_t* x, int T, const int32_t* ids,
                           const float* w, uint16_t* y, int32_t* offsets_out, int32_t* entries_out,
                           uint32_t flags, char* ws, const WsLayout& lay, cudaStream_t st) {
  Control* ctl = reinterpret_cast<Control*>(ws + lay.ctl);
  PfWs p = pf_ws(L, T, ws, lay);
  const int Fmax = L.F > L.Fs ? L.F : L.Fs;
  const int nblk = (T + PF_TOKBLK - 1) / PF_TOKBLK;
  const bool det = (flags & MOE_F_DETERMINISTIC) != 0;
  const int has_shared = L.Fs > 0 ? 1 : 0;
  cudaError_t e = launch_prep_tokens(x, T, L.d, flags, p.xn, p.x16, ctl, st);
  if (e != cudaSuccess) return e;
  if (!det) {
    e = cudaMemsetAsync(p.yacc, 0, (size_t)T * L.d * sizeof(float), st);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(bucket_hist_kernel, dim3(nblk), dim3(256), (size_t)L.E * 4, st, ids, T, L.k, L.E,
                 p.blockcnt, ctl);
  if (e != cudaSuccess) return e;
  e = launch_pdl(bucket_scan_kernel, dim3(1), dim3(1024), 0, st, p.blockcnt, nblk, L.E, T, L.k,
                 has_shared, L.slot, p, offsets_out, ctl);
  if (e != cudaSuccess) return e;
  e = launch_pdl(bucket_scatter_kernel, dim3(nblk), dim3(256), (size_t)L.E * 32, st, ids, w, T, L.k,
                 L.E, has_shared, p, entries_out);
  if (e != cudaSuccess) return e;
  const size_t R = (size_t)T * (L.k + 1);
  e = launch_pdl(gather_rows_kernel, dim3(4 * sm_count()), dim3(256), 0, st,
                 static_cast<const __half*>(p.x16), static_cast<const int*>(p.tokpos),
                 static_cast<const int*>(p.offsets), L.E, T, p.xperm, L.d, ctl);
  if (e != cudaSuccess) return e;
  PfMaps m0, m1;
  memset(&m0, 0, sizeof m0);
  memset(&m1, 0, sizeof m1);
  if (!make_map(&m0.b, p.xperm, (uint64_t)L.d, (uint64_t)R) ||
      !make_map(&m1.b, p.H, (uint64_t)Fmax, (uint64_t)(R + PF_NT)) ||
      !make_code_maps(L, 0, L.codes, L.scales, L.F, L.E, &m0.lo, &m0.hi, &m0.sc) ||
      !make_code_maps(L, 1, L.codes, L.scales, L.F, L.E, &m1.lo, &m1.hi, &m1.sc))
    return cudaErrorInvalidValue;
  if (L.Fs > 0 && (!make_code_maps(L, 0, L.scodes, L.sscales, L.Fs, 1, &m0.slo, &m0.shi, &m0.ssc) ||
                   !make_code_maps(L, 1, L.scodes, L.sscales, L.Fs, 1, &m1.slo, &m1.shi, &m1.ssc)))
    return cudaErrorInvalidValue;
  PfArgs a;
  a.L = L;
  a.T = T;
  a.Fmax = Fmax;
  a.p = p;
  a.det = det ? 1 : 0;
  a.ctl = ctl;
  a.mode = 0;
  a.ppc = (Fmax + 127) / 128;
  e = L.bits == 2 ? launch_gemm<2>(a, m0, st) : launch_gemm<3>(a, m0, st);
  if (e != cudaSuccess) return e;
  a.mode = 1;
  a.ppc = (L.d + 2 * PF_BM - 1) / (2 * PF_BM);
  e = L.bits == 2 ? launch_gemm<2>(a, m1, st) : launch_gemm<3>(a, m1, st);
  if (e != cudaSuccess) return e;
  const long long n4 = (long long)T * L.d / 4;
  int grid = (int)((n4 + 255) / 256);
  if (grid > 4 * sm_count()) grid = 4 * sm_count();
  if (det)
    return launch_pdl(prefill_finalize_det_kernel, dim3(grid), dim3(256), 0, st,
                      static_cast<const float*>(p.ybuf), static_cast<const int*>(p.invpos),
                      static_cast<const int*>(p.offsets), x, T, L.d, L.k, L.E, has_shared, flags, y);
  return launch_pdl(prefill_finalize_kernel, dim3(grid), dim3(256), 0, st,
                    static_cast<const float*>(p.yacc), x, n4, flags, y);
}

}  // namespace moe
