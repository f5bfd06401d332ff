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
//  3. GEMM1:   for each (chunk, 64-feature tile): D[128 x n] = A . B^T where
//              A = 64 gate rows and the 64 matching up rows of the expert,
//              dequantised from the packed 2/3-bit codes into a 128-byte
//              swizzled fp16 tile by producer warps, and B = the chunk's token
//              rows of x16 (gathered with cp.async).  tcgen05.mma accumulates
//              in TMEM; the epilogue reads TMEM, applies SwiGLU and stores the
//              hidden rows H[position][f] (fp16).
//  4. GEMM2:   for each (chunk, 128-row tile of d): D = Wd_tile . H_chunk^T;
//              the epilogue scales column n by its routing weight and adds it
//              into y_acc[token][i] (fp32 reductions).
//  5. finalize y = bf16(y_acc (+ x)).
//
// Warp roles of the GEMM kernel (one CTA per SM, persistent over work items):
//  warps 0-3  epilogue (TMEM lane quadrant = warp index)
//  warps 4-7  A producers: packed codes arrive by bulk copy in a small ring;
//             each thread dequantises one 128-byte row of the A tile
//  warps 8-11 B producers: cp.async of token rows into the swizzled B tile
//  warp 12    TMEM allocation and the single MMA-issuing thread
// Every wait is bounded; a timed-out role records the error and stops waiting.
#include "internal.h"
#include "tc.cuh"

namespace moe {

cudaError_t launch_prep_tokens(const uint16_t* x, int T, int d, uint32_t flags, uint16_t* xn,
                               __half* x16, Control* ctl, cudaStream_t st);

constexpr int PF_NT = 128;        // token tile = MMA N (max)
constexpr int PF_BM = 128;        // MMA M
constexpr int PF_NS = 4;          // operand ring stages
constexpr int PF_CS = 4;          // packed-code ring stages
constexpr int PF_TOKBLK = 256;    // bucketing token block
constexpr int PF_CODE_SLOT = 448; // one 16-row tile in a code stage: lo 256 | hi 128 | scales 64
constexpr int PF_CODE_STAGE = 8 * PF_CODE_SLOT;
constexpr int PF_A_STAGE = PF_BM * 128;
constexpr int PF_B_STAGE = PF_NT * 128;
constexpr int PF_THREADS = 13 * 32;

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
  parts[6] = pf_max_chunks(L, T) * 16 + 256 + R * 4 + 256 + R * 4;   // chunks, tokpos, wpos
  parts[7] = (R + PF_NT) * Fmax * 2;                           // H
  parts[8] = (size_t)T * L.d * 4;                              // yacc
  size_t tot = 0;
  for (int i = 0; i < 9; ++i) tot += parts[i];
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
  p.H = reinterpret_cast<__half*>(ws + lay.h);
  p.yacc = reinterpret_cast<float*>(ws + lay.yacc);
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
                                                           PfWs p, int* __restrict__ user_offsets) {
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
    for (int c = 0; c * PF_NT < cnt[e]; ++c)
      p.chunks[nch[e] + c] = make_int4(e, off[e] + c * PF_NT, min(PF_NT, cnt[e] - c * PF_NT), 0);
  }
  if (tid == 0) {
    p.offsets[E + 1] = off[E] + T;
    p.misc[0] = nchunks;
  }
}

__global__ void __launch_bounds__(256) bucket_scatter_kernel(const int32_t* __restrict__ ids,
                                                             const float* __restrict__ w, int T,
                                                             int k, int E, PfWs p,
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
    if (e < 0 || e >= E) continue;
    int rank = __popc(bits[e * 8 + (lt >> 5)] & ((1u << (lt & 31)) - 1u));
    for (int wd = 0; wd < (lt >> 5); ++wd) rank += __popc(bits[e * 8 + wd]);
    const int pos = p.offsets[e] + p.blockcnt[(size_t)blockIdx.x * E + e] + rank;
    p.entries[pos] = i;
    if (user_entries) user_entries[pos] = i;
    p.tokpos[pos] = t;
    p.wpos[pos] = w[i];
  }
  for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
    const int pos = T * k + t;
    p.tokpos[pos] = t;
    p.wpos[pos] = 1.f;
  }
}

// ----------------------------------------------------------------- GEMM
struct PfArgs {
  LayerDev L;
  int mode;             // 0: gate/up -> H,  1: down -> y_acc
  int T;
  int Fmax;
  int tpc;              // tiles per chunk
  PfWs p;
  const __half* bsrc;   // x16 (mode 0) or H (mode 1)
  int bstride;          // elements per B row
  Control* ctl;
};

struct PfItem {
  int u, pos0, nv, tile, F, K, KS;
  bool valid;
  const uint8_t* codes;
  const uint16_t* scales;
};

__device__ __forceinline__ PfItem pf_item(const PfArgs& a, int i, Control* ctl) {
  PfItem it;
  const int4 ch = a.p.chunks[i / a.tpc];
  it.u = ch.x;
  it.pos0 = ch.y;
  it.nv = ch.z;
  it.tile = i % a.tpc;
  if (it.u >= a.L.E) {
    it.F = a.L.Fs;
    it.codes = a.L.scodes;
    it.scales = a.L.sscales;
  } else {
    int slot = a.L.slot[it.u];
    if (slot < 0 || slot >= a.L.E) {
      record_error(ctl, kErrRange, 0x601);
      slot = 0;
    }
    it.F = a.L.F;
    it.codes = a.L.codes + (long long)slot * a.L.cbe;
    it.scales = a.L.scales + (long long)slot * a.L.nse;
  }
  if (a.mode == 0) {
    it.K = a.L.d;
    it.valid = it.tile * 64 < it.F && it.nv > 0;
  } else {
    it.K = it.F;
    it.valid = it.tile * PF_BM < a.L.d && it.nv > 0 && it.F > 0;
  }
  it.KS = (it.K + 63) / 64;
  return it;
}

// Iterator over this CTA's k-steps: (item, k-step) in the order every role
// walks them.
struct KIter {
  int it, ks, n_items;
  bool done;
  PfItem item;
  __device__ __forceinline__ void next_item(const PfArgs& a, Control* ctl) {
    for (;;) {
      ++it;
      const int i = blockIdx.x + it * gridDim.x;
      if (i >= n_items) {
        done = true;
        return;
      }
      item = pf_item(a, i, ctl);
      if (item.valid) break;
    }
    ks = 0;
  }
  __device__ __forceinline__ void init(const PfArgs& a, int n, Control* ctl) {
    it = -1;
    ks = 0;
    n_items = n;
    done = false;
    next_item(a, ctl);
  }
  __device__ __forceinline__ void advance(const PfArgs& a, Control* ctl) {
    if (++ks >= item.KS) next_item(a, ctl);
  }
};

// Packed-code tile slot q' (0..7) of an A tile: which packed 16-row tile feeds
// it.  Returns false when the slot lies outside the matrix.
__device__ __forceinline__ bool pf_slot(const PfArgs& a, const PfItem& it, int q, const uint8_t** mc,
                                        const uint16_t** ms, int* tau, int* nGK) {
  const int d = a.L.d;
  const long long mcb = mat_codes_bytes(it.F, d, a.L.bits);
  if (a.mode == 0) {
    *tau = 4 * it.tile + (q >> 1);
    *nGK = d / kGroup;
    *mc = it.codes + ((q & 1) ? mcb : 0);
    *ms = it.scales + ((q & 1) ? (long long)it.F * (d / kGroup) : 0);
    return *tau < it.F / kTileRows;
  }
  *tau = 8 * it.tile + q;
  *nGK = it.F / kGroup;
  *mc = it.codes + 2 * mcb;
  *ms = it.scales + 2LL * it.F * (d / kGroup);
  return *tau < d / kTileRows;
}

// warp-cooperative: bulk-copy the packed codes of k-step ks of `it` into a code stage
__device__ __forceinline__ void pf_issue_codes(const PfArgs& a, const PfItem& it, int ks,
                                               unsigned char* stage, uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const int bits = a.L.bits;
  const int gbase = 2 * ks;
  const int ng = min(2, it.K / kGroup - gbase);
  uint32_t total = 0;
  for (int q = 0; q < 8; ++q) {
    const uint8_t* mc;
    const uint16_t* ms;
    int tau, nGK;
    if (pf_slot(a, it, q, &mc, &ms, &tau, &nGK)) total += ng * (128 + 32 + (bits == 3 ? 64 : 0));
  }
  if (lane == 0) mbar_arrive_expect_tx(bar, total);
  __syncwarp();
  if (lane < 24) {
    const int q = lane / 3, part = lane % 3;
    const uint8_t* mc;
    const uint16_t* ms;
    int tau, nGK;
    if (pf_slot(a, it, q, &mc, &ms, &tau, &nGK)) {
      const long long tcb = (long long)nGK * kTileRows * group_bytes(bits);
      unsigned char* dst = stage + q * PF_CODE_SLOT;
      if (part == 0) {
        bulk_g2s(dst, mc + tau * tcb + gbase * 128, ng * 128, bar);
      } else if (part == 1) {
        if (bits == 3) bulk_g2s(dst + 256, mc + tau * tcb + nGK * 128 + gbase * 64, ng * 64, bar);
      } else {
        bulk_g2s(dst + 384, ms + (long long)tau * kTileRows * nGK + gbase * 16, ng * 32, bar);
      }
    }
  }
}

// dequantise chunk m (8 consecutive K values) of one group into fp16
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

struct PfSmem {
  size_t a, b, codes, bars, holder, total;
};
__host__ __device__ inline PfSmem pf_smem() {
  PfSmem m;
  size_t o = 0;
  m.a = o;
  o += (size_t)PF_NS * PF_A_STAGE;
  m.b = o;
  o += (size_t)PF_NS * PF_B_STAGE;
  m.codes = o;
  o += (size_t)PF_CS * PF_CODE_STAGE;
  m.bars = o;
  o += (2 * PF_NS + PF_CS + 4) * 8;
  m.holder = o;
  o += 16;
  m.total = o + 1024;   // slack to align the base to 1024
  return m;
}

template <int BITS>
__global__ void __launch_bounds__(PF_THREADS, 1) pf_gemm_kernel(const PfArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const PfSmem m = pf_smem();
  unsigned char* sA = smem + m.a;
  unsigned char* sB = smem + m.b;
  unsigned char* sC = smem + m.codes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + m.bars);
  uint64_t* empty = full + PF_NS;
  uint64_t* cfull = empty + PF_NS;
  uint64_t* tfull = cfull + PF_CS;
  uint64_t* tempty = tfull + 2;
  uint32_t* holder = reinterpret_cast<uint32_t*>(smem + m.holder);
  Control* ctl = a.ctl;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < PF_NS; ++s) {
      mbar_init(&full[s], 256);
      mbar_init(&empty[s], 1);
    }
    for (int c = 0; c < PF_CS; ++c) mbar_init(&cfull[c], 1);
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
  pdl_wait();
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *holder;
  const int n_items = a.p.misc[0] * a.tpc;
  bool ok = true;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------ A producers (dequant)
    const int r = tid - 128;
    KIter ahead;   // issuer's iterator, PF_CS k-steps ahead
    if (warp == 4) {
      ahead.init(a, n_items, ctl);
      for (int c = 0; c < PF_CS && !ahead.done; ++c) {
        pf_issue_codes(a, ahead.item, ahead.ks, sC + c * PF_CODE_STAGE, &cfull[c]);
        ahead.advance(a, ctl);
      }
    }
    KIter cur;
    cur.init(a, n_items, ctl);
    int g = 0;
    while (!cur.done) {
      const PfItem& it = cur.item;
      const int cs = g % PF_CS;
      if (ok) ok = mbar_wait(&cfull[cs], (g / PF_CS) & 1, ctl, 0x610);
      const unsigned char* cst = sC + cs * PF_CODE_STAGE;
      int q, rr;
      if (a.mode == 0) {
        q = 2 * (r >> 5) + (((r & 31) >> 4) & 1);
        rr = r & 15;
      } else {
        q = r >> 4;
        rr = r & 15;
      }
      const uint8_t* mc;
      const uint16_t* ms;
      int tau, nGK;
      const bool rv = pf_slot(a, it, q, &mc, &ms, &tau, &nGK);
      const int ng = min(2, it.K / kGroup - 2 * cur.ks);
      uint4 chunk[8];
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        uint32_t X[4], Y[4];
        __half2 s2 = __float2half2_rn(0.f);
        if (rv && gi < ng && ok) {
          const unsigned char* slot = cst + q * PF_CODE_SLOT;
          const uint2 lo = *reinterpret_cast<const uint2*>(slot + (gi * 16 + rr) * 8);
          const uint32_t hi = BITS == 3 ? *reinterpret_cast<const uint32_t*>(slot + 256 + (gi * 16 + rr) * 4) : 0u;
          const __half s = *reinterpret_cast<const __half*>(slot + 384 + (gi * 16 + rr) * 2);
          s2 = __half2half2(s);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            X[t] = __byte_perm(lo.x, lo.y, (uint32_t)t | ((uint32_t)(4 + t) << 8));
            Y[t] = hi >> (4 * t);
          }
        } else {
#pragma unroll
          for (int t = 0; t < 4; ++t) X[t] = Y[t] = 0u;
        }
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) chunk[gi * 4 + mm] = pf_dq_chunk<BITS>(X, Y, mm, s2);
      }
      named_bar_sync(2, 128);   // every A thread has read code stage cs
      if (warp == 4 && !ahead.done) {
        pf_issue_codes(a, ahead.item, ahead.ks, sC + cs * PF_CODE_STAGE, &cfull[cs]);
        ahead.advance(a, ctl);
      }
      const int s = g % PF_NS;
      if (g >= PF_NS && ok) ok = mbar_wait(&empty[s], ((g / PF_NS) - 1) & 1, ctl, 0x611);
      unsigned char* at = sA + s * PF_A_STAGE + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(at + ((c ^ (r & 7)) << 4)) = chunk[c];
      fence_proxy_async_smem();
      mbar_arrive(&full[s]);
      cur.advance(a, ctl);
      ++g;
    }
  } else if (warp >= 8 && warp < 12) {
    // ------------------------------------------------ B producers (rows)
    const int b = tid - 256;
    const int c = b & 7;
    KIter cur;
    cur.init(a, n_items, ctl);
    int g = 0, prev_s = -1;
    const __half* rows[8];
    int cur_it = -1;
    while (!cur.done) {
      const PfItem& it = cur.item;
      const int n_mma = (it.nv + 15) & ~15;
      if (cur.it != cur_it) {
        cur_it = cur.it;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int n = (b >> 3) + 16 * i;
          rows[i] = a.bsrc;
          if (n < it.nv) {
            const int row = a.mode == 0 ? a.p.tokpos[it.pos0 + n] : it.pos0 + n;
            rows[i] = a.bsrc + (size_t)row * a.bstride;
          }
        }
      }
      const int s = g % PF_NS;
      if (g >= PF_NS && ok) ok = mbar_wait(&empty[s], ((g / PF_NS) - 1) & 1, ctl, 0x620);
      const int nc = 4 * min(2, it.K / kGroup - 2 * cur.ks);
      unsigned char* bt = sB + s * PF_B_STAGE;
      if (c < nc && ok) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int n = (b >> 3) + 16 * i;
          if (n < n_mma)
            cp_async16(bt + n * 128 + ((c ^ (n & 7)) << 4), rows[i] + 64 * cur.ks + 8 * c,
                       n < it.nv ? 16u : 0u);
        }
      }
      cp_async_commit();
      if (prev_s >= 0) {
        cp_async_wait<1>();
        fence_proxy_async_smem();
        mbar_arrive(&full[prev_s]);
      }
      prev_s = s;
      cur.advance(a, ctl);
      ++g;
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    if (prev_s >= 0) mbar_arrive(&full[prev_s]);
  } else if (warp == 12) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      KIter cur;
      cur.init(a, n_items, ctl);
      int g = 0, la = 0;
      while (!cur.done) {
        const PfItem it = cur.item;
        const int acc = la & 1;
        if (la >= 2 && ok) ok = mbar_wait(&tempty[acc], ((la >> 1) - 1) & 1, ctl, 0x630);
        tc_fence_after();
        const int n_mma = (it.nv + 15) & ~15;
        const uint32_t idesc = idesc_f16_f32(PF_BM, n_mma);
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        for (int ks = 0; ks < it.KS; ++ks) {
          const int s = g % PF_NS;
          if (ok) ok = mbar_wait(&full[s], (g / PF_NS) & 1, ctl, 0x631);
          tc_fence_after();
          const int nk = 2 * min(2, it.K / kGroup - 2 * ks);
          const uint32_t abase = smem_u32(sA + s * PF_A_STAGE);
          const uint32_t bbase = smem_u32(sB + s * PF_B_STAGE);
          if (ok) {
            for (int kk = 0; kk < nk; ++kk)
              tc_mma_f16(d_tmem, sw128_kmajor_desc(abase + kk * 32), sw128_kmajor_desc(bbase + kk * 32),
                         idesc, (ks | kk) != 0);
          }
          tc_commit(&empty[s]);
          ++g;
        }
        tc_commit(&tfull[acc]);
        ++la;
        cur.next_item(a, ctl);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 0-3)
    const int q = warp;
    KIter cur;
    cur.init(a, n_items, ctl);
    int la = 0;
    while (!cur.done) {
      const PfItem it = cur.item;
      const int acc = la & 1;
      if (ok) ok = mbar_wait(&tfull[acc], (la >> 1) & 1, ctl, 0x640);
      tc_fence_after();
      const int n_mma = (it.nv + 15) & ~15;
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * 256);
      if (a.mode == 0) {
        const int f = 64 * it.tile + 16 * q + (lane & 15);
        const bool wr = lane < 16 && f < it.F;
        for (int c0 = 0; c0 < n_mma; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float gv = __uint_as_float(v[j]);
            const float up = __shfl_xor_sync(0xffffffffu, gv, 16);
            const int n = c0 + j;
            if (wr && n < it.nv && ok) {
              const float h = gv / (1.f + expf(-gv)) * up;
              a.p.H[(size_t)(it.pos0 + n) * a.Fmax + f] = __float2half_rn(h);
            }
          }
        }
      } else {
        const int i_out = PF_BM * it.tile + 32 * q + lane;
        const bool wr = i_out < a.L.d;
        for (int c0 = 0; c0 < n_mma; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int n = c0 + j;
            if (wr && n < it.nv && ok) {
              const int tok = a.p.tokpos[it.pos0 + n];
              const float wv = a.p.wpos[it.pos0 + n];
              atomicAdd(a.p.yacc + (size_t)tok * a.L.d + i_out, __uint_as_float(v[j]) * wv);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      ++la;
      cur.next_item(a, ctl);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 12) tmem_dealloc(tmem_base, 512);
}

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

template <int BITS>
static cudaError_t launch_gemm(const PfArgs& a, cudaStream_t st) {
  const PfSmem m = pf_smem();
  cudaError_t e = cudaFuncSetAttribute(pf_gemm_kernel<BITS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)m.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(pf_gemm_kernel<BITS>, dim3(sm_count()), dim3(PF_THREADS), m.total, st, a);
}

cudaError_t launch_prefill(const LayerDev& L, const uint16_t* x, int T, const int32_t* ids,
                           const float* w, uint16_t* y, int32_t* offsets_out, int32_t* entries_out,
                           uint32_t flags, char* ws, const WsLayout& lay, cudaStream_t st) {
  Control* ctl = reinterpret_cast<Control*>(ws + lay.ctl);
  PfWs p = pf_ws(L, T, ws, lay);
  const int Fmax = L.F > L.Fs ? L.F : L.Fs;
  const int nblk = (T + PF_TOKBLK - 1) / PF_TOKBLK;
  cudaError_t e = launch_prep_tokens(x, T, L.d, flags, p.xn, p.x16, ctl, st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(p.yacc, 0, (size_t)T * L.d * sizeof(float), st);
  if (e != cudaSuccess) return e;
  e = launch_pdl(bucket_hist_kernel, dim3(nblk), dim3(256), (size_t)L.E * 4, st, ids, T, L.k, L.E,
                 p.blockcnt, ctl);
  if (e != cudaSuccess) return e;
  e = launch_pdl(bucket_scan_kernel, dim3(1), dim3(1024), 0, st, p.blockcnt, nblk, L.E, T, L.k,
                 L.Fs > 0 ? 1 : 0, p, offsets_out);
  if (e != cudaSuccess) return e;
  e = launch_pdl(bucket_scatter_kernel, dim3(nblk), dim3(256), (size_t)L.E * 32, st, ids, w, T, L.k,
                 L.E, p, entries_out);
  if (e != cudaSuccess) return e;
  PfArgs a;
  a.L = L;
  a.T = T;
  a.Fmax = Fmax;
  a.p = p;
  a.mode = 0;
  a.tpc = (Fmax + 63) / 64;
  a.bsrc = p.x16;
  a.bstride = L.d;
  a.ctl = ctl;
  e = L.bits == 2 ? launch_gemm<2>(a, st) : launch_gemm<3>(a, st);
  if (e != cudaSuccess) return e;
  a.mode = 1;
  a.tpc = (L.d + PF_BM - 1) / PF_BM;
  a.bsrc = p.H;
  a.bstride = Fmax;
  e = L.bits == 2 ? launch_gemm<2>(a, st) : launch_gemm<3>(a, st);
  if (e != cudaSuccess) return e;
  const long long n4 = (long long)T * L.d / 4;
  int grid = (int)((n4 + 255) / 256);
  if (grid > 4 * sm_count()) grid = 4 * sm_count();
  return launch_pdl(prefill_finalize_kernel, dim3(grid), dim3(256), 0, st,
                    static_cast<const float*>(p.yacc), x, n4, flags, y);
}

}  // namespace moe
