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
//              and stores it as row `position` of ybuf (fp16, plain coalesced
//              stores: no float atomics).
//  6. combine: y[t] = bf16(sum of the ybuf rows of token t in selection order,
//              shared expert last (+ x)): a fixed order, so prefill output does
//              not depend on scheduling.
//
// Warp roles of the GEMM kernel (one CTA per SM, persistent over work items):
//  warps 0-3   epilogue (TMEM lane quadrant = warp index)
//  warps 4-11  A producers in two groups of four warps; group j fills the A
//              stages of the k-steps g with g % 2 == j, so two k-steps are
//              dequantised at once.  A thread loads the packed codes of one
//              32-value group of two rows of both tiles (one group k-step
//              ahead, into registers) and writes them dequantised, swizzled.
//  warp 12     TMEM allocation; one elected lane issues the MMAs
//  warp 13     loads: the B tile of every k-step by TMA (rows of the permuted
//              token buffer, or of H) into the k-step ring, and each item's
//              packed codes into L2 (bulk prefetch) one item ahead
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
constexpr int PF_NS = 4;          // k-step ring stages: an A tile pair (dequantised on chip)
                                  // and a B tile (TMA) share one full and one empty barrier
constexpr int PF_TOKBLK = 256;    // bucketing token block
constexpr int PF_A_TILE = PF_BM * 128;     // one 128 x 64 fp16 tile
constexpr int PF_A_STAGE = 2 * PF_A_TILE;  // a tile pair
constexpr int PF_B_STAGE = PF_NT * 128;
constexpr int PF_THREADS = 14 * 32;
constexpr int PF_A_WARPS = 4;      // warps of one producer group (two groups)

struct PfWs {
  int* counts;      // [E+1]
  int* misc;        // [16]: misc[0] = number of chunks
  int* offsets;     // [E+2]: padded bucket offsets (internal positions)
  int* uoffsets;    // [E+2]: bucket offsets without padding (user-visible)
  int* entries;     // [T*k]
  int* blockcnt;    // [nblk][E]
  int4* chunks;     // [maxC]
  int* tokpos;      // [T*(k+1)]
  float* wpos;      // [T*(k+1)]
  __half* H;        // [(T*(k+1) + 128)][Fmax]
  __half* x16;      // [T][d]
  uint16_t* xn;     // [T][d]
  int* invpos;      // [T*k]: position of entry t*k+j in the buckets (-1: invalid id)
  __half* xperm;    // [T*(k+1)][d]: token rows in bucket order (GEMM1 operand)
  __half* ybuf;     // [T*(k+1)][d]: weighted expert rows (GEMM2 output), aliases xperm
};

// Internal positions: every bucket starts at a multiple of PF_PAD rows (so that
// whole 32-row blocks of a chunk stay inside its bucket); the padding rows
// carry token -1.  At most min(E, T*k) + 1 buckets are non-empty.
constexpr int PF_PAD = 32;
static size_t pf_rows(const LayerDev& L, int T) {
  const size_t nonempty = (size_t)((long long)T * L.k < L.E ? (long long)T * L.k : L.E) + 1;
  return (size_t)T * (L.k + 1) + (size_t)PF_PAD * nonempty;
}

static size_t pf_max_chunks(const LayerDev& L, int T) {
  return (size_t)T * L.k / PF_NT + L.E + (T + PF_NT - 1) / PF_NT + 2;
}

size_t prefill_ws_bytes(const LayerDev& L, int T, size_t* parts) {
  const int Fmax = L.F > L.Fs ? L.F : L.Fs;
  const size_t nblk = ((size_t)T + PF_TOKBLK - 1) / PF_TOKBLK;
  const size_t R = pf_rows(L, T);
  parts[0] = (size_t)T * L.d * 2;                              // xn
  parts[1] = (size_t)T * L.d * 2;                              // x16
  parts[2] = (size_t)(L.E + 1 + 16) * 4;                       // counts + misc
  parts[3] = 2 * (size_t)(L.E + 2) * 4;                        // offsets, uoffsets
  parts[4] = (size_t)T * L.k * 4;                              // entries
  parts[5] = nblk * L.E * 4;                                   // blockcnt
  parts[6] = pf_max_chunks(L, T) * 16 + 256 + 2 * (R * 4 + 256) + (size_t)T * L.k * 4;
                                                               // chunks, tokpos, wpos, invpos
  parts[7] = (R + PF_NT) * Fmax * 2;                           // H
  parts[8] = 0;                                                // (unused)
  parts[9] = R * L.d * 2;                                      // xperm / ybuf
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
  p.uoffsets = p.offsets + (L.E + 2);
  p.entries = reinterpret_cast<int*>(ws + lay.entries);
  p.blockcnt = reinterpret_cast<int*>(ws + lay.blockcnt);
  char* t = ws + lay.tiles;
  p.chunks = reinterpret_cast<int4*>(t);
  t += (pf_max_chunks(L, T) * 16 + 255) / 256 * 256;
  p.tokpos = reinterpret_cast<int*>(t);
  const size_t R = pf_rows(L, T);
  t += (R * 4 + 255) / 256 * 256;
  p.wpos = reinterpret_cast<float*>(t);
  t += (R * 4 + 255) / 256 * 256;
  p.invpos = reinterpret_cast<int*>(t);
  p.H = reinterpret_cast<__half*>(ws + lay.h);
  p.xperm = reinterpret_cast<__half*>(ws + lay.xperm);
  p.ybuf = reinterpret_cast<__half*>(ws + lay.xperm);
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
  __shared__ int cnt[2048], off[2048], poff[2048], nch[2048], wt[33];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  // per expert, the exclusive running sum over token blocks; the block
  // counts are loaded 16 at a time so that their latencies overlap
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
    for (int b0 = 0; b0 < nblk; b0 += 16) {
      int c[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) c[j] = b0 + j < nblk ? blockcnt[(size_t)(b0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (b0 + j < nblk) blockcnt[(size_t)(b0 + j) * E + e] = run;
        run += c[j];
      }
    }
    cnt[e] = run;
  }
  if (tid == 0) cnt[E] = has_shared ? T : 0;   // the shared expert: every token
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) {
    off[e] = cnt[e];
    poff[e] = (cnt[e] + PF_PAD - 1) / PF_PAD * PF_PAD;
    nch[e] = (cnt[e] + PF_NT - 1) / PF_NT;
  }
  __syncthreads();
  block_excl_scan(off, E + 1, wt);
  block_excl_scan(poff, E + 1, wt);
  const int nchunks = block_excl_scan(nch, E + 1, wt);
  for (int e = tid; e <= E; e += blockDim.x) {
    p.counts[e] = cnt[e];
    p.offsets[e] = poff[e];
    p.uoffsets[e] = off[e];
    if (user_offsets) user_offsets[e] = off[e];
    for (int r = cnt[e]; r % PF_PAD; ++r) p.tokpos[poff[e] + r] = -1;   // padding rows
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
      p.chunks[nch[e] + c] = make_int4(e, poff[e] + c * PF_NT, min(PF_NT, cnt[e] - c * PF_NT), s);
  }
  if (tid == 0) {
    p.offsets[E + 1] = poff[E] + (cnt[E] + PF_PAD - 1) / PF_PAD * PF_PAD;
    p.uoffsets[E + 1] = off[E] + cnt[E];
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
    const int before = p.blockcnt[(size_t)blockIdx.x * E + e] + rank;
    const int pos = p.offsets[e] + before, upos = p.uoffsets[e] + before;
    p.entries[upos] = i;
    p.invpos[i] = pos;
    if (user_entries) user_entries[upos] = i;
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
// positions pos < offsets[E+1] (routed buckets, then the shared bucket; the
// padding rows are skipped).  One warp per row, 16-byte accesses, four in
// flight per lane.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __half* __restrict__ x16,
                                                          const int* __restrict__ tokpos,
                                                          const int* __restrict__ offsets, int E,
                                                          int T, __half* __restrict__ xperm,
                                                          int d, Control* ctl) {
  pdl_wait();
  pdl_launch_dependents();
  const int per = d / 8;   // 16-byte pieces of a row
  const int lane = threadIdx.x & 31;
  const int nrows = offsets[E + 1];
  const int nw = gridDim.x * (blockDim.x >> 5);
  bool bad = false;
  for (int pos = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); pos < nrows; pos += nw) {
    int t = tokpos[pos];
    if (t < 0) continue;   // padding row
    if (t >= T) {
      bad = true;
      t = 0;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x16 + (size_t)t * d);
    uint4* dst = reinterpret_cast<uint4*>(xperm + (size_t)pos * d);
    for (int c0 = lane; c0 < per; c0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + 32 * u < per) v[u] = src[c0 + 32 * u];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + 32 * u < per) dst[c0 + 32 * u] = v[u];
    }
  }
  if (bad && lane == 0) record_error(ctl, kErrRange, 0x602);
}

// ----------------------------------------------------------------- GEMM
struct PfArgs {
  LayerDev L;
  int mode;     // 0: gate/up -> H,  1: down -> ybuf
  int T;
  int Fmax;
  int ppc;      // tile pairs (work items) per chunk
  int debug;    // MOE_F_DEBUG given: the control block's test switch is honoured
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

// Tensor map of the B operand: token rows of xperm (mode 0) or hidden rows of
// H (mode 1).
struct alignas(64) PfMaps {
  CUtensorMap b;
  CUtensorMap st;   // epilogue output: H (mode 0, box 64 x 32) or ybuf (mode 1, box 128 x 32)
};

// 32 output rows of one tile (staged in shared memory) to global memory by TMA.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Read-only global loads that do not allocate in L1 (the packed codes are read
// once per CTA; reuse across CTAs is served by L2).  Volatile so that they stay
// ahead of the waits that follow them in program order.
__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_nc_u16(const void* p) {
  unsigned short v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ void l2_prefetch_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Geometry of the matrices a work item reads: the codes and scales of its
// expert (slot, or the shared expert), the code bytes of a 16-row tile and the
// groups along K.
struct PfGeo {
  const uint8_t* codes;     // matrix of mode 1 (Wd) / Wg of mode 0
  const uint16_t* scales;
  long long up_codes;       // mode 0: Wu codes - Wg codes (bytes)
  long long up_scales;      // mode 0: Wu scales - Wg scales (elements)
  int tcb, nG, rows_blk;    // code bytes per 16-row tile, groups along K, 16-row tiles
};

template <int BITS>
__device__ __forceinline__ PfGeo pf_geo(const PfArgs& a, const PfItem& it) {
  PfGeo g;
  constexpr int gb = BITS == 2 ? 8 : 12;
  const uint8_t* ec = it.shared ? a.L.scodes : a.L.codes + (long long)it.slot * a.L.cbe;
  const uint16_t* es = it.shared ? a.L.sscales : a.L.scales + (long long)it.slot * a.L.nse;
  const int nGd = a.L.d / kGroup;
  const long long tcbd = (long long)nGd * kTileRows * gb;   // Wg / Wu tile bytes
  if (a.mode == 0) {
    g.codes = ec;
    g.scales = es;
    g.up_codes = (long long)(it.F / kTileRows) * tcbd;
    g.up_scales = (long long)it.F * nGd;
    g.tcb = (int)tcbd;
    g.nG = nGd;
    g.rows_blk = it.F / kTileRows;
  } else {
    g.codes = ec + 2 * (long long)(it.F / kTileRows) * tcbd;
    g.scales = es + 2 * (long long)it.F * nGd;
    g.up_codes = 0;
    g.up_scales = 0;
    g.nG = it.F / kGroup;
    g.tcb = g.nG * kTileRows * gb;
    g.rows_blk = a.L.d / kTileRows;
  }
  return g;
}

// One lane: bring the packed codes and scales an item will read into L2.
template <int BITS>
__device__ __forceinline__ void pf_prefetch_item(const PfArgs& a, const PfItem& it) {
  const PfGeo g = pf_geo<BITS>(a, it);
  const int per = a.mode == 0 ? 8 : 16;                 // 16-row tiles of a pair, per matrix
  const int b0 = per * it.pair;
  const int nb = min(per, g.rows_blk - b0);
  if (nb <= 0) return;
  const uint32_t cb = (uint32_t)nb * g.tcb, sb = (uint32_t)nb * g.nG * kTileRows * 2;
  const uint8_t* c = g.codes + (long long)b0 * g.tcb;
  const uint16_t* sc = g.scales + (long long)b0 * g.nG * kTileRows;
  l2_prefetch_bulk(c, cb);
  l2_prefetch_bulk(sc, sb);
  if (a.mode == 0) {
    l2_prefetch_bulk(c + g.up_codes, cb);
    l2_prefetch_bulk(sc + g.up_scales, sb);
  }
}

// The packed codes of one producer thread for one k-step: four units (row rq
// or rq + 64 of tile 0 or 1, one 32-value group), loaded into registers one
// group k-step ahead of their use.
struct PfRaw {
  uint2 lo[4];
  uint32_t hi[4];
  uint32_t sc[4];
  uint32_t meta;   // bits 0-3: unit u present; bits 4-5: groups in the k-step
};

// Per-item addresses of a producer thread's four units: the 16-row tile of
// each unit (codes and scales), computed once per work item.
struct PfUnits {
  const uint8_t* tb[4];
  const uint16_t* sb[4];
  uint32_t mask;   // units whose rows are inside the matrix
  int hioff;       // start of the high-bit plane within a tile (bytes)
  int key;         // the item these addresses belong to (-1: none)
};

template <int BITS>
__device__ __forceinline__ void pf_units(const PfArgs& a, const PfItem& it, int rq, PfUnits& U) {
  const PfGeo g = pf_geo<BITS>(a, it);
  int blk, dblk, rblk;
  const uint8_t* mc = g.codes;
  const uint16_t* ms = g.scales;
  if (a.mode == 0) {
    // A-tile rows: four blocks of [16 gate rows, 16 up rows]
    const int qt = rq >> 5, isu = (rq >> 4) & 1;
    blk = 8 * it.pair + qt;
    dblk = 4;
    rblk = 2;
    if (isu) {
      mc += g.up_codes;
      ms += g.up_scales;
    }
  } else {
    blk = 16 * it.pair + (rq >> 4);
    dblk = 8;
    rblk = 4;
  }
  uint32_t mask = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int b = blk + (u >> 1) * dblk + (u & 1) * rblk;
    const bool in = b < g.rows_blk && ((u >> 1) == 0 || it.two);
    U.tb[u] = mc + (long long)(in ? b : 0) * g.tcb;
    U.sb[u] = ms + (long long)(in ? b : 0) * g.nG * kTileRows;
    mask |= in ? 1u << u : 0u;
  }
  U.mask = mask;
  U.hioff = g.nG * 128;
}

template <int BITS>
__device__ __forceinline__ void pf_load_raw(const PfArgs& a, const KSeq& q, int rq, int gi,
                                            PfUnits& U, PfRaw& r) {
  const PfItem& it = q.item_ref();
  if (U.key != q.s.i) {
    pf_units<BITS>(a, it, rq, U);
    U.key = q.s.i;
  }
  const int ng = q.ks == it.KS - 1 ? it.ng_last : 2;
  const int w = (2 * q.ks + gi) * kTileRows + (rq & 15);   // word (group, row) within a tile
  const uint32_t use = gi < ng ? U.mask : 0u;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    if ((use >> u) & 1u) {
      r.lo[u] = ldg_nc_v2(U.tb[u] + w * 8);
      r.hi[u] = BITS == 3 ? ldg_nc_u32(U.tb[u] + U.hioff + w * 4) : 0u;
      r.sc[u] = ldg_nc_u16(U.sb[u] + w);
    } else {
      r.lo[u] = make_uint2(0u, 0u);
      r.hi[u] = 0u;
      r.sc[u] = 0u;
    }
  }
  r.meta = ((uint32_t)ng << 4) | use;
}

// Dequantise chunk m (8 consecutive K values) of one group into fp16.  The
// code q of a value sits in a half's mantissa under the exponent of 1024
// (magic 0x6400), scaled by 4^-m for its bit position; one fma recentres it
// to q - 2^(b-1) exactly, and the multiply by the fp16 scale is the only
// rounding step.
template <int BITS>
__device__ __forceinline__ uint4 pf_dq_chunk(const uint32_t (&X)[4], const uint32_t (&Y)[4], int m,
                                             __half2 s2) {
  // fp16 constants as bit patterns (both halves): 4^-m, and the recentring
  // terms -(1024 + 2) 4^-m (2-bit); for 3 bits the high plane's 2^(2-m) and
  // -(1024 * 2^(2-m) + 4 + 1024 * 4^-m)
  constexpr uint32_t kMulR[4] = {0x3C003C00u, 0x34003400u, 0x2C002C00u, 0x24002400u};
  constexpr uint32_t kAddR2[4] = {0xE402E402u, 0xDC08DC08u, 0xD420D420u, 0xCC80CC80u};
  constexpr uint32_t kMulH[4] = {0x44004400u, 0x40004000u, 0x3C003C00u, 0x38003800u};
  constexpr uint32_t kAddH[4] = {0xED01ED01u, 0xE882E882u, 0xE444E444u, 0xE028E028u};
  const uint32_t magic = 0x64006400u;
  const uint32_t mask = 0x00030003u << (2 * m);
  uint32_t out[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const __half2 R = u32_as_h2(and_or(X[t], mask, magic));
    __half2 v;
    if (BITS == 2) {
      v = __hfma2(R, u32_as_h2(kMulR[m]), u32_as_h2(kAddR2[m]));
    } else {
      const __half2 H = u32_as_h2(and_or(Y[t], 0x00010001u << m, magic));
      const __half2 tmp = __hfma2(H, u32_as_h2(kMulH[m]), u32_as_h2(kAddH[m]));
      v = __hfma2(R, u32_as_h2(kMulR[m]), tmp);
    }
    out[t] = h2_as_u32(__hmul2(v, s2));
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

constexpr int PF_OUT_STAGE = 32 * 128 * 2;   // 32 rows x 128 fp16 (mode 1); mode 0 uses 32 x 64
struct PfSmem {
  size_t a, b, out, bars, holder, total;
};
__host__ __device__ inline PfSmem pf_smem() {
  PfSmem m;
  size_t o = 0;
  m.a = o;
  o += (size_t)PF_NS * PF_A_STAGE;
  m.b = o;
  o += (size_t)PF_NS * PF_B_STAGE;
  m.out = o;                       // epilogue staging: two 32-row blocks
  o += 2 * (size_t)PF_OUT_STAGE;
  m.bars = o;
  o += (3 * PF_NS + 5) * 8;
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
  unsigned char* sOut = smem + m.out;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + m.bars);   // A: 4 producer warps
  uint64_t* bfull = full + PF_NS;                                  // B: the TMA load
  uint64_t* empty = bfull + PF_NS;                                 // MMA commit
  uint64_t* tfull = empty + PF_NS;
  uint64_t* tempty = tfull + 2;
  uint64_t* mdone = tempty + 2;                                    // every MMA issued has completed
  uint32_t* holder = reinterpret_cast<uint32_t*>(smem + m.holder);
  Control* ctl = a.ctl;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < PF_NS; ++s) {
      mbar_init(&full[s], PF_A_WARPS);
      mbar_init(&bfull[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
    }
    mbar_init(mdone, 1);
    fence_barrier_init();
  }
  if (warp == 12) {
    tmem_alloc(holder, 512);
    tmem_relinquish();
  }
  if (warp == 13 && lane < 2)   // the tensor-map descriptors into the TMA unit's cache
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(lane ? &mp.st : &mp.b))
                 : "memory");
  pdl_wait();
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *holder;
  const int n_items = a.p.misc[0] * a.ppc;
  // Give-up rule: a role whose bounded wait runs out (the timeout is recorded
  // in the error word) stops issuing copies, MMAs, stores and arrives, and
  // leaves its loop; the decision is uniform over the warp (over the four
  // epilogue warps for the epilogue).  Before the CTA releases its TMEM and
  // shared memory, the loader waits for every copy it issued and the MMA
  // issuer for every MMA it issued, so nothing asynchronous is in flight when
  // the CTA ends.  The roles left waiting on a role that gave up run out in
  // turn, so a stuck pipeline ends within a few wait limits.
  bool ok = true;

  if (warp >= 4 && warp < 12) {
    // ------------------------------------------------ A producers (dequant)
    // Group grp = k-step parity.  Thread = (group gi of the k-step, rows rq and
    // rq + 64 of both tiles): four 32-value units per k-step, whose packed
    // codes are loaded one group k-step (two k-steps) ahead.
    const int grp = (warp - 4) >> 2;
    const int ta = tid - 128 - 128 * grp;
    const int rq = ta >> 1, gi = ta & 1;
    // swizzled 16-byte chunk offsets of this thread's group in a row
    uint32_t swz[4];
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) swz[mm] = (uint32_t)(((4 * gi + mm) ^ (rq & 7)) << 4);
    unsigned char* const adst = sA + rq * 128;
    KSeq q;
    q.init(a, n_items);
    if (grp == 1 && !q.done) q.advance(a);
    // Rotating register buffers: no copy of a buffer ever waits on its loads.
    // Returns false when the wait for the stage ran out.
    auto produce = [&](const PfRaw& r, int g) -> bool {
      const int sa = g % PF_NS;
      if (g >= PF_NS) {
        ok = __all_sync(0xffffffffu, mbar_wait(&empty[sa], ((g / PF_NS) - 1) & 1, ctl, 0x611));
        if (!ok) return false;
      }
      if (gi < (int)(r.meta >> 4)) {
        // unit u: tile u >> 1 (+16 KB), row rq + 64 (u & 1) (+8 KB); absent
        // units (rows outside the matrix) are written as zeros
        unsigned char* at = adst + sa * PF_A_STAGE;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t X[4], Y[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            X[t] = __byte_perm(r.lo[u].x, r.lo[u].y, (uint32_t)t | ((uint32_t)(4 + t) << 8));
            Y[t] = r.hi[u] >> (4 * t);
          }
          const __half2 s2 = __half2half2(__ushort_as_half((unsigned short)r.sc[u]));
#pragma unroll
          for (int mm = 0; mm < 4; ++mm)
            *reinterpret_cast<uint4*>(at + (u >> 1) * PF_A_TILE + (u & 1) * 8192 + swz[mm]) =
                pf_dq_chunk<BITS>(X, Y, mm, s2);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[sa]);
      return true;
    };
    auto skip2 = [&]() {   // this group's next k-step
      q.advance(a);
      if (!q.done) q.advance(a);
    };
    PfRaw r0, r1, r2;
    PfUnits U;
    U.key = -1;
    // three buffers: the codes of the group's next two k-steps are in flight
    // while the current one is dequantised
    bool h0 = false, h1 = false, h2 = false;
    if (!q.done) {
      pf_load_raw<BITS>(a, q, rq, gi, U, r0);
      skip2();
      h0 = true;
    }
    if (!q.done) {
      pf_load_raw<BITS>(a, q, rq, gi, U, r1);
      skip2();
      h1 = true;
    }
    int g = grp;
    for (;;) {
      if (!h0) break;
      h2 = !q.done;
      if (h2) {
        pf_load_raw<BITS>(a, q, rq, gi, U, r2);
        skip2();
      }
      if (!produce(r0, g)) break;
      g += 2;
      if (!h1) break;
      h0 = !q.done;
      if (h0) {
        pf_load_raw<BITS>(a, q, rq, gi, U, r0);
        skip2();
      }
      if (!produce(r1, g)) break;
      g += 2;
      if (!h2) break;
      h1 = !q.done;
      if (h1) {
        pf_load_raw<BITS>(a, q, rq, gi, U, r1);
        skip2();
      }
      if (!produce(r2, g)) break;
      g += 2;
    }
  } else if (warp == 13) {
    // ------------------------------------------------ loads: B by TMA, codes into L2
    // The whole warp walks the loop; one elected lane issues.
    const bool leader = elect_one();
    ItemSeq pfs;
    pfs.init(a, n_items);
    PfItem pit;
    bool have = pfs.get(a, pit);
    if (have && leader) pf_prefetch_item<BITS>(a, pit);
    have = have && pfs.get(a, pit);
    KSeq cur;
    cur.init(a, n_items);
    int g = 0, sb = 0;
    uint32_t pb = 0;
    while (!cur.done) {
      if (cur.ks == 0 && g > 0 && have) {   // a new item: codes of the one after it
        if (leader) pf_prefetch_item<BITS>(a, pit);
        have = pfs.get(a, pit);
      }
      if (g >= PF_NS) {
        ok = __all_sync(0xffffffffu, mbar_wait(&empty[sb], pb ^ 1u, ctl, 0x620));
        if (!ok) break;
      }
      if (leader) {
        mbar_arrive_expect_tx(&bfull[sb], PF_B_STAGE);
        tma_load_2d(sB + sb * PF_B_STAGE, &mp.b, 64 * cur.ks, cur.item_ref().pos0, &bfull[sb]);
      }
      __syncwarp();
      if (++sb == PF_NS) {
        sb = 0;
        pb ^= 1u;
      }
      cur.advance(a);
      ++g;
    }
    // The last min(g, PF_NS) copies, one per stage and each its stage's newest
    // phase, may not have been consumed (always the case after a give-up
    // anywhere in the CTA): wait for them to land.  On the normal path they
    // have landed already.
    if (leader)
      for (int j = g > PF_NS ? g - PF_NS : 0; j < g; ++j)
        mbar_wait(&bfull[j % PF_NS], (uint32_t)(j / PF_NS) & 1u, ctl, 0x621);
    __syncwarp();
  } else if (warp == 12) {
    // ------------------------------------------------ MMA issuer
    // The whole warp walks the loop (its values stay warp-uniform); one
    // elected lane issues the MMAs and the commits.
    const bool leader = elect_one();
    const uint64_t adesc0 = sw128_kmajor_desc(smem_u32(sA));
    const uint64_t bdesc0 = sw128_kmajor_desc(smem_u32(sB));
    ItemSeq seq;
    seq.init(a, n_items);
    PfItem it;
    int s = 0, la = 0;
    uint32_t ph = 0;
    bool issued = false;
    while (seq.get(a, it)) {
      const int acc = la & 1;
      if (la >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&tempty[acc], ((la >> 1) - 1) & 1, ctl, 0x630));
        if (!ok) break;
      }
      tc_fence_after();
      const uint32_t idesc = idesc_f16_f32(PF_BM, (it.nv + 15) & ~15);
      const uint32_t d0 = tmem_base + (uint32_t)(acc * 256), d1 = d0 + 128;
      const bool two = it.two;
      for (int ks = 0; ks < it.KS; ++ks) {
        // B (one TMA load) lands long before the dequantised A tile: its
        // wait is passed by the time A's completes
        bool got = mbar_wait(&bfull[s], ph, ctl, 0x632);
        got = got && mbar_wait(&full[s], ph, ctl, 0x631);
        ok = __all_sync(0xffffffffu, got);
        if (!ok) break;
        tc_fence_after();
        const uint64_t ad = adesc0 + (uint64_t)(s * (PF_A_STAGE >> 4));
        const uint64_t bd = bdesc0 + (uint64_t)(s * (PF_B_STAGE >> 4));
        const uint32_t first = ks > 0 ? 1u : 0u;
        const bool full = ks < it.KS - 1 || it.ng_last == 2;
        if (leader) {
          tc_mma_f16(d0, ad, bd, idesc, first);
          tc_mma_f16(d0, ad + 2, bd + 2, idesc, 1u);
          if (two) {
            tc_mma_f16(d1, ad + (PF_A_TILE >> 4), bd, idesc, first);
            tc_mma_f16(d1, ad + (PF_A_TILE >> 4) + 2, bd + 2, idesc, 1u);
          }
          if (full) {
            tc_mma_f16(d0, ad + 4, bd + 4, idesc, 1u);
            tc_mma_f16(d0, ad + 6, bd + 6, idesc, 1u);
            if (two) {
              tc_mma_f16(d1, ad + (PF_A_TILE >> 4) + 4, bd + 4, idesc, 1u);
              tc_mma_f16(d1, ad + (PF_A_TILE >> 4) + 6, bd + 6, idesc, 1u);
            }
          }
          tc_commit(&empty[s]);
        }
        issued = true;
        __syncwarp();
        if (++s == PF_NS) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      if (leader) tc_commit(&tfull[acc]);
      __syncwarp();
      ++la;
    }
    // every MMA issued has completed before the CTA releases its TMEM
    if (issued) {
      if (leader) tc_commit(mdone);
      __syncwarp();
      mbar_wait(mdone, 0, ctl, 0x633);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 0-3)
    // Each 32-column block of an accumulator tile becomes 32 output rows,
    // staged in shared memory (two buffers) and written by one TMA store; the
    // rows past the chunk's tokens are padding rows of the same bucket.
    const int q = warp;
    ItemSeq seq;
    seq.init(a, n_items);
    PfItem it;
    int la = 0, cc = 0;
    // test switch: thread 0 of block 0 of the gate/up GEMM keeps back its
    // arrive on the first accumulator's barrier, so the MMA issuer's wait
    // before its third item runs out (held here, not in the producer warps,
    // which are the pipeline's bottleneck)
    const bool withhold =
        a.debug && a.mode == 0 && blockIdx.x == 0 && tid == 0 &&
        *reinterpret_cast<volatile uint32_t*>(&ctl->debug_withhold) == kWithholdPrefillArrive;
    // free a staging buffer (the store issued from it two blocks ago has read it)
    auto claim = [&]() {
      if (tid == 0 && cc >= 2) bulk_wait_read<1>();
      named_bar_sync(3, 128);
    };
    auto release = [&](int x0, int row0) {
      fence_proxy_async_smem();
      named_bar_sync(3, 128);
      if (tid == 0) {
        tma_store_2d(&mp.st, sOut + (cc & 1) * PF_OUT_STAGE, x0, row0);
        bulk_commit();
      }
      ++cc;
    };
    while (seq.get(a, it)) {
      const int acc = la & 1;
      // mode 1: routing weights of this item's columns (lane + 32 c)
      float wcol[4] = {0.f, 0.f, 0.f, 0.f};
      if (a.mode == 1) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (lane + 32 * c < it.nv) wcol[c] = a.p.wpos[it.pos0 + lane + 32 * c];
      }
      ok = mbar_wait(&tfull[acc], (la >> 1) & 1, ctl, 0x640);
      if (named_bar_any(3, 128, !ok)) {   // one epilogue thread gave up: all four warps stop
        ok = false;
        break;
      }
      tc_fence_after();
      const int n_mma = (it.nv + 15) & ~15;
      const int ntile = it.two ? 2 : 1;
      for (int v = 0; v < ntile; ++v) {
        const uint32_t taddr =
            tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * 256 + v * 128);
        for (int c0 = 0; c0 < n_mma; c0 += 32) {
          uint32_t rv[32];
          tmem_ld_32x32b_x32(taddr + c0, rv);
          tmem_ld_wait();
          if (v == ntile - 1 && c0 + 32 >= n_mma) {
            tc_fence_before();
            if (!(withhold && la == 0)) mbar_arrive(&tempty[acc]);   // TMEM free: item + 2 may start
          }
          claim();
          __half* so = reinterpret_cast<__half*>(sOut + (cc & 1) * PF_OUT_STAGE);
          if (a.mode == 0) {
            // SwiGLU: TMEM lane 32q + l holds gate row 16q + l (l < 16) or the
            // matching up row (l >= 16); a step pairs two token columns so that
            // every lane computes one output.  Stage [32 rows][64 f].
            const int hi = lane >> 4, fl = 16 * q + (lane & 15);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float a0 = __uint_as_float(rv[j]), a1 = __uint_as_float(rv[j + 1]);
              const float got = __shfl_xor_sync(0xffffffffu, hi ? a0 : a1, 16);
              const float gv = hi ? got : a0;
              const float up = hi ? a1 : got;
              so[(j + hi) * 64 + fl] = __float2half_rn(__fdividef(gv * up, 1.f + __expf(-gv)));
            }
            release(64 * (2 * it.pair + v), it.pos0 + c0);
          } else {
            // weighted rows of the down projection: stage [32 rows][128 d]
            const float wl = c0 == 0 ? wcol[0] : (c0 == 32 ? wcol[1] : (c0 == 64 ? wcol[2] : wcol[3]));
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float wj = __shfl_sync(0xffffffffu, wl, j);
              so[j * 128 + 32 * q + lane] = __float2half_rn(__uint_as_float(rv[j]) * wj);
            }
            release(PF_BM * (2 * it.pair + v), it.pos0 + c0);
          }
        }
      }
      ++la;
    }
    if (tid == 0) bulk_wait<0>();   // every output row written before the CTA leaves
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 12) tmem_dealloc(tmem_base, 512);
}

// Combine: y[t] = bf16(sum over j = 0..k-1 of ybuf[invpos[t][j]] + ybuf[shared
// row of t] (+ x[t])), the routed terms in selection order and the shared
// expert last, in fp32; every term already carries its routing weight.  The
// fixed order makes the result independent of scheduling.  One warp per
// token, 8 elements (16 bytes of fp16) per lane and step; the terms' loads
// are issued four at a time (their positions staged in shared memory), so
// their latencies overlap while the sum keeps its order.
__global__ void __launch_bounds__(256) prefill_combine_kernel(
    const __half* __restrict__ ybuf, const int* __restrict__ invpos, const int* __restrict__ offsets,
    const uint16_t* __restrict__ x, int T, int d, int k, int E, int has_shared, uint32_t flags,
    uint16_t* __restrict__ y) {
  __shared__ int spos[8][17];   // per warp: the token's k routed positions, then the shared one
  pdl_wait();
  pdl_launch_dependents();
  const int per = d / 8;
  const int sh0 = offsets[E];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int nw = gridDim.x * (blockDim.x >> 5);
  const int nt = k + 1;
  for (int t = blockIdx.x * (blockDim.x >> 5) + wib; t < T; t += nw) {
    __syncwarp();
    if (lane < k) spos[wib][lane] = invpos[(size_t)t * k + lane];
    if (lane == 0) spos[wib][k] = has_shared ? sh0 + t : -1;
    __syncwarp();
    for (int c = lane; c < per; c += 32) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
      // the terms in a fixed order (selection order, shared expert last; -1:
      // no term), loaded four at a time so that their latencies overlap
      for (int j0 = 0; j0 < nt; j0 += 4) {
        uint4 u[4];
        int pq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          pq[q] = j0 + q < nt ? spos[wib][j0 + q] : -1;
          u[q] = pq[q] >= 0 ? reinterpret_cast<const uint4*>(ybuf + (size_t)pq[q] * d)[c]
                            : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (pq[q] < 0) continue;
          const uint32_t w4[4] = {u[q].x, u[q].y, u[q].z, u[q].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(u32_as_h2(w4[e]));
            v[2 * e] += f.x;
            v[2 * e + 1] += f.y;
          }
        }
      }
      const size_t i = (size_t)t * per + c;
      if (flags & MOE_F_RESIDUAL) {
        const uint4 xv = reinterpret_cast<const uint4*>(x)[i];
        const uint32_t x4[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[2 * e] += __uint_as_float(x4[e] << 16);
          v[2 * e + 1] += __uint_as_float(x4[e] & 0xFFFF0000u);
        }
      }
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        o[e] = *reinterpret_cast<uint32_t*>(&b2);
      }
      reinterpret_cast<uint4*>(y)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
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

// 2-D 16-bit row-major tensor [rows][inner] (fp16 or bf16: the copy moves
// bytes) for tiles of 128 rows x 64 elements, 128-byte swizzle (the canonical
// K-major UMMA layout).
// 2-D 16-bit row-major tensor [rows][inner], box [box_rows][box_inner], no
// swizzle (the epilogue's output stores).
static bool make_map_b16_plain(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                               uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_b16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows) {
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
  const int has_shared = L.Fs > 0 ? 1 : 0;
  cudaError_t e = launch_prep_tokens(x, T, L.d, flags, p.xn, p.x16, ctl, st);
  if (e != cudaSuccess) return e;
  e = launch_pdl(bucket_hist_kernel, dim3(nblk), dim3(256), (size_t)L.E * 4, st, ids, T, L.k, L.E,
                 p.blockcnt, ctl);
  if (e != cudaSuccess) return e;
  e = launch_pdl(bucket_scan_kernel, dim3(1), dim3(1024), 0, st, p.blockcnt, nblk, L.E, T, L.k,
                 has_shared, L.slot, p, offsets_out, ctl);
  if (e != cudaSuccess) return e;
  e = launch_pdl(bucket_scatter_kernel, dim3(nblk), dim3(256), (size_t)L.E * 32, st, ids, w, T, L.k,
                 L.E, has_shared, p, entries_out);
  if (e != cudaSuccess) return e;
  const size_t R = pf_rows(L, T);
  e = launch_pdl(gather_rows_kernel, dim3(4 * sm_count()), dim3(256), 0, st,
                 static_cast<const __half*>(p.x16), static_cast<const int*>(p.tokpos),
                 static_cast<const int*>(p.offsets), L.E, T, p.xperm, L.d, ctl);
  if (e != cudaSuccess) return e;
  PfMaps m0, m1;
  memset(&m0, 0, sizeof m0);
  memset(&m1, 0, sizeof m1);
  if (!make_map_b16(&m0.b, p.xperm, (uint64_t)L.d, (uint64_t)R) ||
      !make_map_b16(&m1.b, p.H, (uint64_t)Fmax, (uint64_t)(R + PF_NT)) ||
      !make_map_b16_plain(&m0.st, p.H, (uint64_t)Fmax, (uint64_t)(R + PF_NT), 64, 32) ||
      !make_map_b16_plain(&m1.st, p.ybuf, (uint64_t)L.d, (uint64_t)R, 128, 32))
    return cudaErrorInvalidValue;
  PfArgs a;
  a.L = L;
  a.T = T;
  a.Fmax = Fmax;
  a.p = p;
  a.ctl = ctl;
  a.debug = (flags & MOE_F_DEBUG) ? 1 : 0;
  a.mode = 0;
  a.ppc = (Fmax + 127) / 128;
  e = L.bits == 2 ? launch_gemm<2>(a, m0, st) : launch_gemm<3>(a, m0, st);
  if (e != cudaSuccess) return e;
  a.mode = 1;
  a.ppc = (L.d + 2 * PF_BM - 1) / (2 * PF_BM);
  e = L.bits == 2 ? launch_gemm<2>(a, m1, st) : launch_gemm<3>(a, m1, st);
  if (e != cudaSuccess) return e;
  int grid = (T + 7) / 8;
  if (grid > 4 * sm_count()) grid = 4 * sm_count();
  return launch_pdl(prefill_combine_kernel, dim3(grid), dim3(256), 0, st,
                    static_cast<const __half*>(p.ybuf), static_cast<const int*>(p.invpos),
                    static_cast<const int*>(p.offsets), x, T, L.d, L.k, L.E, has_shared, flags, y);
}

}  // namespace moe
