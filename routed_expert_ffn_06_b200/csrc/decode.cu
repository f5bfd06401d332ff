// decode.cu -- decode / verify-window expert step (T <= 8 tokens).
//
// "Checking several tokens costs little more than writing one: the common
// weights are read once and only the experts the extra tokens route to add
// work" ("Why Strata is fast on low-VRAM GPUs", section "guess first, then
// check").  So the window's selected experts are deduplicated and every
// selected expert's packed weights are streamed from HBM exactly once per call.
//
// Two kernels, chained with programmatic dependent launch (PDL):
//  * decode_gu: work item = (expert u, 16-row tile of Wg and Wu).  A quad of
//    four warps shares an item: each warp takes pieces of 16 quantisation
//    groups of the K = d contraction, streams them into its own shared-memory
//    stages with warp-wide cp.async, dequantises the 2/3-bit codes straight into
//    mma.sync A fragments (LOP3 + HFMA2: no shared-memory round trip for the
//    fp16 weights) and multiplies them with the window's tokens (B fragments;
//    n = 8 covers T <= 8).  The quad adds its partial sums through shared
//    memory, applies SwiGLU and the routing weight and writes
//    hw[u][f][t] = w_u[t] * silu(g) * up  (fp16, in B-fragment order).
//  * decode_dn: one CTA per 16-row tile of the output.  Its Wd tiles depend
//    only on the routing, so they are requested before the kernel waits for
//    decode_gu; the hidden vectors follow after the wait.  Warps sum over the
//    experts, then the CTA adds the warps in a fixed order (deterministic, no
//    atomics) and writes y (bf16, optional residual).
// The shared expert is expert u = 0 with weight 1 for every token.
// Each warp owns its stages and fills them itself (gate/up: cp.async groups;
// down: bulk copies on per-stage mbarriers, every wait on the current phase).
#include "internal.h"
#include "tc.cuh"

namespace moe {

constexpr int kMaxExp = kMaxDecodeT * 16 + 1;   // window entries + shared
constexpr int kGuWarps = 16;                 // four quads
constexpr int kDnWarps = 16;

struct ExpList {
  int n;                       // experts in the list (shared first when present)
  int id[kMaxExp];             // expert id, -1 = shared
  int slot[kMaxExp];           // packed-weight slot of the expert
  float w[kMaxExp][kMaxDecodeT];
  int uidx[kMaxDecodeT * 16];  // list position of a window entry's expert
};

// All threads: the expert -> slot table into shared memory (it does not depend
// on earlier kernels) and the list's weight table cleared.  Out-of-range slots
// are replaced by 0 and flagged, so no later address leaves the expert array.
__device__ void expert_list_prologue(const LayerDev& L, ExpList* s, int* slot_s, int* first,
                                     Control* ctl) {
  for (int e = threadIdx.x; e < L.E; e += blockDim.x) {
    int sl = L.slot[e];
    if (sl < 0 || sl >= L.E) {
      record_error(ctl, kErrRange, 0x301);
      sl = 0;
    }
    slot_s[e] = sl;
    first[e] = 0x7FFFFFFF;
  }
  for (int i = threadIdx.x; i < kMaxExp * kMaxDecodeT; i += blockDim.x) (&s->w[0][0])[i] = 0.f;
}

// Warp 0 (after expert_list_prologue and a block barrier): deduplicate the
// window's T*k selections in first-occurrence order.  Out-of-range ids are
// dropped and flagged.
__device__ void build_expert_list(const int32_t* __restrict__ ids, const float* __restrict__ w,
                                  int T, const LayerDev& L, ExpList* s, const int* slot_s,
                                  int* first, Control* ctl) {
  const int lane = threadIdx.x & 31;
  const int n_ent = T * L.k;
  const int base = L.Fs > 0 ? 1 : 0;
  int ent[4];
  float entw[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int i = lane + 32 * c;
    ent[c] = i < n_ent ? ids[i] : -1;
    entw[c] = i < n_ent ? w[i] : 0.f;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int i = lane + 32 * c;
    if (i < n_ent) {
      if (ent[c] < 0 || ent[c] >= L.E) {
        record_error(ctl, kErrRange, 0x300);
        ent[c] = -1;
      } else {
        atomicMin(&first[ent[c]], i);
      }
    }
  }
  __syncwarp();
  int count = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int i = lane + 32 * c;
    const bool f = i < n_ent && ent[c] >= 0 && first[ent[c]] == i;
    const unsigned mask = __ballot_sync(0xffffffffu, f);
    if (f) {
      const int pos = base + count + __popc(mask & ((1u << lane) - 1u));
      s->id[pos] = ent[c];
      s->slot[pos] = slot_s[ent[c]];
      s->uidx[i] = pos;
    }
    count += __popc(mask);
  }
  __syncwarp();
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int i = lane + 32 * c;
    if (i < n_ent && ent[c] >= 0) {
      const int u = s->uidx[first[ent[c]]];
      atomicAdd(&s->w[u][i / L.k], entw[c]);
    }
  }
  if (lane == 0) {
    s->n = base + count;
    if (base) {
      s->id[0] = -1;
      s->slot[0] = 0;
      for (int t = 0; t < kMaxDecodeT; ++t) s->w[0][t] = t < T ? 1.f : 0.f;
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------ dequant to A
// 2-bit: the 8-byte group word of one row -> four fp16x2 A registers holding
// (code - 2) for columns 8m + 2t + {0,1}, m = 0..3 (t = lane % 4).
__device__ __forceinline__ void dq2(uint2 lo, uint32_t sel, uint32_t (&a)[4]) {
  const uint32_t X = __byte_perm(lo.x, lo.y, sel);
  const uint32_t magic = 0x64006400u;  // fp16 1024 in both halves
  a[0] = h2_as_u32(__hfma2(u32_as_h2(and_or(X, 0x00030003u, magic)), __float2half2_rn(1.f),
                           __float2half2_rn(-1026.f)));
  a[1] = h2_as_u32(__hfma2(u32_as_h2(and_or(X, 0x000C000Cu, magic)), __float2half2_rn(0.25f),
                           __float2half2_rn(-258.f)));
  a[2] = h2_as_u32(__hfma2(u32_as_h2(and_or(X, 0x00300030u, magic)), __float2half2_rn(0.0625f),
                           __float2half2_rn(-66.f)));
  a[3] = h2_as_u32(__hfma2(u32_as_h2(and_or(X, 0x00C000C0u, magic)), __float2half2_rn(0.015625f),
                           __float2half2_rn(-18.f)));
}

// 3-bit: low planes as above plus the 4-byte high-bit word; (code - 4).
__device__ __forceinline__ void dq3(uint2 lo, uint32_t hi, uint32_t sel, uint32_t hshift,
                                    uint32_t (&a)[4]) {
  const uint32_t X = __byte_perm(lo.x, lo.y, sel);
  const uint32_t Y = hi >> hshift;
  const uint32_t magic = 0x64006400u;
  __half2 t;
  t = __hfma2(u32_as_h2(and_or(Y, 0x00010001u, magic)), __float2half2_rn(4.f),
              __float2half2_rn(-5124.f));
  a[0] = h2_as_u32(__hfma2(u32_as_h2(and_or(X, 0x00030003u, magic)), __float2half2_rn(1.f), t));
  t = __hfma2(u32_as_h2(and_or(Y, 0x00020002u, magic)), __float2half2_rn(2.f),
              __float2half2_rn(-2308.f));
  a[1] = h2_as_u32(__hfma2(u32_as_h2(and_or(X, 0x000C000Cu, magic)), __float2half2_rn(0.25f), t));
  t = __hfma2(u32_as_h2(and_or(Y, 0x00040004u, magic)), __float2half2_rn(1.f),
              __float2half2_rn(-1092.f));
  a[2] = h2_as_u32(__hfma2(u32_as_h2(and_or(X, 0x00300030u, magic)), __float2half2_rn(0.0625f), t));
  t = __hfma2(u32_as_h2(and_or(Y, 0x00080008u, magic)), __float2half2_rn(0.5f),
              __float2half2_rn(-532.f));
  a[3] = h2_as_u32(__hfma2(u32_as_h2(and_or(X, 0x00C000C0u, magic)), __float2half2_rn(0.015625f), t));
}

// One 16-row x 32-column group of a packed tile times the B fragments of that
// group: acc += scale_row * (A_group . B).  lo: the tile's 8-byte words
// (group-major, word (c, r) at (c*16 + r)*8), hi: its 4-byte high-bit words
// (3-bit), sc: its scales (element c*16 + r).
template <int BITS>
__device__ __forceinline__ void group_mma(const unsigned char* lo, const unsigned char* hi,
                                          const __half* sc, int c, const uint32_t (&b)[4],
                                          float (&acc)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint32_t sel = (uint32_t)t | ((uint32_t)(4 + t) << 8);
  const uint2 lo0 = *reinterpret_cast<const uint2*>(lo + (c * 16 + g) * 8);
  const uint2 lo1 = *reinterpret_cast<const uint2*>(lo + (c * 16 + g + 8) * 8);
  uint32_t a0[4], a1[4];
  if (BITS == 2) {
    dq2(lo0, sel, a0);
    dq2(lo1, sel, a1);
  } else {
    const uint32_t h0 = *reinterpret_cast<const uint32_t*>(hi + (c * 16 + g) * 4);
    const uint32_t h1 = *reinterpret_cast<const uint32_t*>(hi + (c * 16 + g + 8) * 4);
    dq3(lo0, h0, sel, 4 * t, a0);
    dq3(lo1, h1, sel, 4 * t, a1);
  }
  const float zero[4] = {0.f, 0.f, 0.f, 0.f};
  float tmp[4];
  const uint32_t A0[4] = {a0[0], a1[0], a0[1], a1[1]};
  const uint32_t B0[2] = {b[0], b[1]};
  mma_f16_16816(tmp, A0, B0, zero);
  const uint32_t A1[4] = {a0[2], a1[2], a0[3], a1[3]};
  const uint32_t B1[2] = {b[2], b[3]};
  mma_f16_16816(tmp, A1, B1, tmp);
  const float s0 = __half2float(sc[c * 16 + g]);
  const float s1 = __half2float(sc[c * 16 + g + 8]);
  acc[0] = fmaf(s0, tmp[0], acc[0]);
  acc[1] = fmaf(s0, tmp[1], acc[1]);
  acc[2] = fmaf(s1, tmp[2], acc[2]);
  acc[3] = fmaf(s1, tmp[3], acc[3]);
}

// 2-bit group MMA without per-weight arithmetic beyond one LOP3: the A
// fragment holds the raw fp16 value 1024 + 4^m*q of each code (the magic-number
// trick), the B fragment holds the token value divided by 4^m (exact power-of-
// two scaling, done once when the tokens are staged), so A*B = 1024*B + q*x.
// The term sum_k B_k*(1024 + 2*4^m_k), precomputed per (token, group) from the
// same fp16 B values, enters as the negated C input of the first MMA, leaving
// sum_k (q_k - 2)*x_k for the group; the scale is applied in fp32.
__device__ __forceinline__ void group_mma_2b_offset(const unsigned char* lo, const __half* sc,
                                                    int c, const uint32_t (&b)[4], float2 corr,
                                                    float (&acc)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint32_t sel = (uint32_t)t | ((uint32_t)(4 + t) << 8);
  const uint2 lo0 = *reinterpret_cast<const uint2*>(lo + (c * 16 + g) * 8);
  const uint2 lo1 = *reinterpret_cast<const uint2*>(lo + (c * 16 + g + 8) * 8);
  const uint32_t X0 = __byte_perm(lo0.x, lo0.y, sel), X1 = __byte_perm(lo1.x, lo1.y, sel);
  const uint32_t magic = 0x64006400u;
  const uint32_t A0[4] = {and_or(X0, 0x00030003u, magic), and_or(X1, 0x00030003u, magic),
                          and_or(X0, 0x000C000Cu, magic), and_or(X1, 0x000C000Cu, magic)};
  const uint32_t A1[4] = {and_or(X0, 0x00300030u, magic), and_or(X1, 0x00300030u, magic),
                          and_or(X0, 0x00C000C0u, magic), and_or(X1, 0x00C000C0u, magic)};
  const float cinit[4] = {-corr.x, -corr.y, -corr.x, -corr.y};
  float tmp[4];
  const uint32_t B0[2] = {b[0], b[1]};
  mma_f16_16816(tmp, A0, B0, cinit);
  const uint32_t B1[2] = {b[2], b[3]};
  mma_f16_16816(tmp, A1, B1, tmp);
  const float s0 = __half2float(sc[c * 16 + g]);
  const float s1 = __half2float(sc[c * 16 + g + 8]);
  acc[0] = fmaf(s0, tmp[0], acc[0]);
  acc[1] = fmaf(s0, tmp[1], acc[1]);
  acc[2] = fmaf(s1, tmp[2], acc[2]);
  acc[3] = fmaf(s1, tmp[3], acc[3]);
}

// Source of expert u (shared when u == 0 and the layer has one).
struct ExpSrc {
  const uint8_t* codes;
  const uint16_t* scales;
  int F;
};
__device__ __forceinline__ ExpSrc expert_src(const LayerDev& L, const ExpList* s, int u,
                                             Control* ctl) {
  ExpSrc r;
  (void)ctl;
  if (s->id[u] < 0) {
    r.codes = L.scodes;
    r.scales = L.sscales;
    r.F = L.Fs;
  } else {
    const int slot = s->slot[u];
    r.codes = L.codes + (long long)slot * L.cbe;
    r.scales = L.scales + (long long)slot * L.nse;
    r.F = L.F;
  }
  return r;
}

// ------------------------------------------------------------------ gate/up
// hw layout (fp16): [u][c = f/32][lane < 4T][8 halves] -- the B fragments of
// the down projection for the T real tokens, so a CTA can bulk-copy one
// expert's hidden vector (2*F*T bytes) in one piece.
__host__ __device__ inline size_t hw_expert_halves(int Fmax, int T) { return (size_t)Fmax * T; }

constexpr int kGuPiece = 16;                 // groups per piece of a gate/up item
struct GuSmem {
  size_t bars, list, first, xs, corr, part, stages, total, stage_bytes;
  int spw;                                   // stages per warp
};
__host__ __device__ inline size_t gu_stage_bytes(int bits) {
  // Wg lo | Wg hi | Wu lo | Wu hi | Wg scales | Wu scales   (one piece)
  const size_t lo = kGuPiece * kTileRows * 8, hi = bits == 3 ? kGuPiece * kTileRows * 4 : 0;
  return 2 * (lo + hi) + 2 * kGuPiece * kTileRows * 2;
}
__host__ __device__ inline GuSmem gu_smem(int d, int E, int bits, int spw) {
  GuSmem m;
  const int nG = d / kGroup;
  size_t o = 0;
  m.spw = spw;
  m.bars = o;
  o += (size_t)kGuWarps * spw * sizeof(uint64_t);
  o = (o + 15) & ~size_t(15);
  m.list = o;
  o += sizeof(ExpList);
  o = (o + 15) & ~size_t(15);
  m.first = o;
  o += 2 * (size_t)E * sizeof(int);   // first-occurrence scratch, slot table
  o = (o + 127) & ~size_t(127);
  m.xs = o;
  o += (size_t)nG * 32 * 16;
  m.corr = o;                                // [group][token] fp32 (2-bit offset form)
  o += (size_t)nG * kMaxDecodeT * sizeof(float);
  m.part = o;                                // [quad][2][warp in quad][lane][8] floats
  o += (size_t)(kGuWarps / 4) * 2 * 4 * 32 * 8 * sizeof(float);
  o = (o + 127) & ~size_t(127);
  m.stages = o;
  m.stage_bytes = gu_stage_bytes(bits);
  o += (size_t)kGuWarps * spw * m.stage_bytes;
  m.total = o;
  return m;
}

__device__ __forceinline__ void gu_item(const LayerDev& L, int i, int Fs16, int F16, int* u,
                                        int* tile) {
  if (i < Fs16) {
    *u = 0;
    *tile = i;
  } else {
    *u = (L.Fs > 0 ? 1 : 0) + (i - Fs16) / F16;
    *tile = (i - Fs16) % F16;
  }
}

// Warp-wide copy of `bytes` (a multiple of 16, both ends 16-byte aligned) from
// global to shared memory, 16 bytes per lane and instruction (cp.async: many
// small pieces in flight without going through the bulk-copy unit).
__device__ __forceinline__ void warp_cp_async(void* dst, const void* src, uint32_t bytes) {
  const int lane = threadIdx.x & 31;
  for (uint32_t o = (uint32_t)lane * 16; o < bytes; o += 512)
    cp_async16(static_cast<unsigned char*>(dst) + o, static_cast<const unsigned char*>(src) + o, 16);
}
// Wait until at most n of this thread's cp.async groups are pending (n <= 3).
__device__ __forceinline__ void cp_async_wait_upto(int n) {
  if (n <= 0)
    cp_async_wait<0>();
  else if (n == 1)
    cp_async_wait<1>();
  else if (n == 2)
    cp_async_wait<2>();
  else
    cp_async_wait<3>();
}

// Piece p (groups kGuPiece*p onwards) of gate/up item (u, tile) into a stage, by
// the whole warp: one cp.async group.
template <int BITS>
__device__ __forceinline__ void gu_copy(const LayerDev& L, const ExpList* list, int u, int tile,
                                        int p, unsigned char* st, Control* ctl) {
  const int d = L.d, nG = d / kGroup;
  const int g0 = kGuPiece * p, np = min(kGuPiece, nG - g0);
  const ExpSrc src = expert_src(L, list, u, ctl);
  const long long tcb = (long long)nG * kTileRows * group_bytes(BITS);
  const long long mcb = mat_codes_bytes(src.F, d, BITS);
  const long long msc = (long long)src.F * nG;
  const uint32_t blo = np * kTileRows * 8, bhi = BITS == 3 ? np * kTileRows * 4 : 0;
  const uint32_t bsc = np * kTileRows * 2;
  const size_t LO = kGuPiece * kTileRows * 8, HI = BITS == 3 ? kGuPiece * kTileRows * 4 : 0;
#pragma unroll
  for (int mat = 0; mat < 2; ++mat) {
    const uint8_t* tb = src.codes + (mat ? mcb : 0) + tile * tcb;
    unsigned char* so = st + mat * (LO + HI);
    warp_cp_async(so, tb + g0 * kTileRows * 8, blo);
    if (BITS == 3) warp_cp_async(so + LO, tb + (long long)nG * kTileRows * 8 + g0 * kTileRows * 4, bhi);
    const uint16_t* sb = src.scales + (mat ? msc : 0) + (long long)tile * kTileRows * nG;
    warp_cp_async(st + 2 * (LO + HI) + mat * kGuPiece * kTileRows * 2, sb + g0 * kTileRows, bsc);
  }
  cp_async_commit();
}

template <int BITS>
__global__ void __launch_bounds__(kGuWarps * 32, 1)
    decode_gu_kernel(LayerDev L, const uint16_t* __restrict__ x, int T,
                     const int32_t* __restrict__ ids, const float* __restrict__ wts,
                     __half* __restrict__ hw, int Fmax, uint32_t flags, Control* ctl, int spw) {
  extern __shared__ __align__(128) unsigned char smem[];
  const GuSmem m = gu_smem(L.d, L.E, BITS, spw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + m.bars);
  ExpList* list = reinterpret_cast<ExpList*>(smem + m.list);
  int* first = reinterpret_cast<int*>(smem + m.first);
  uint4* xs = reinterpret_cast<uint4*>(smem + m.xs);
  float* corr = reinterpret_cast<float*>(smem + m.corr);
  float* part = reinterpret_cast<float*>(smem + m.part);
  __shared__ float inv_rms[kMaxDecodeT];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nthreads = kGuWarps * 32;
  const int d = L.d, nG = d / kGroup;
  if (tid == 0) {
    for (int s = 0; s < kGuWarps * spw; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  if (tid == 32) {
    // the next layer's router and shared expert into L2: an equal 16-byte
    // aligned slice of each range per CTA (constant data, so before the wait)
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      const unsigned B = L.pfb[r];
      const unsigned chunk = ((B + gridDim.x - 1) / gridDim.x + 15u) & ~15u;
      const unsigned lo = chunk * blockIdx.x;
      if (lo < B) prefetch_l2(L.pf[r] + lo, B - lo < chunk ? B - lo : chunk);
    }
  }
  expert_list_prologue(L, list, first + L.E, first, ctl);
  // ---- tokens -> B fragments.  x is an input of the whole block: readable
  //      before this grid waits on the router.
  if (warp < T && (flags & MOE_F_PRENORM)) {
    float ss = 0.f;
#pragma unroll 4
    for (int i = lane * 8; i < d; i += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(x + (size_t)warp * d + i);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a = __uint_as_float(w4[j] << 16), b = __uint_as_float(w4[j] & 0xFFFF0000u);
        ss += a * a + b * b;
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) inv_rms[warp] = rsqrtf(ss / (float)d + 1e-6f);
  }
  __syncthreads();
  // one (token n, group c) pair per thread: 32 values -> the 16-byte B
  // fragments of lanes 4n .. 4n+3 (pair m of lane 4n+t = columns 8m+2t, +1)
  for (int pidx = tid; pidx < kMaxDecodeT * nG; pidx += nthreads) {
    const int c = pidx >> 3, n = pidx & 7;
    uint4 out[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                    make_uint4(0, 0, 0, 0)};
    if (n < T) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)n * d + 32 * c);
      uint32_t w[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = src[q];
        w[4 * q] = v.x;
        w[4 * q + 1] = v.y;
        w[4 * q + 2] = v.z;
        w[4 * q + 3] = v.w;
      }
      const bool pn = flags & MOE_F_PRENORM;
      const float sc = pn ? inv_rms[n] : 1.f;
      uint32_t h2[16];
      float cs = 0.f;
      bool bad = false;
#pragma unroll
      for (int q = 0; q < 16; ++q) {   // w[q] holds columns 2q, 2q+1 = 8m + 2t (+1), q = 4m + t
        float v0 = __uint_as_float(w[q] << 16), v1 = __uint_as_float(w[q] & 0xFFFF0000u);
        if (pn) {
          v0 = __bfloat162float(__float2bfloat16_rn(v0 * sc));
          v1 = __bfloat162float(__float2bfloat16_rn(v1 * sc));
        }
        // fp16 operands: values outside the fp16 range are flagged (always on)
        bad |= !(fabsf(v0) <= 65504.f) || !(fabsf(v1) <= 65504.f);
        if (BITS == 2) {
          // offset form: B = x / 4^m; correction sum B * (1024 + 2 * 4^m)
          const float inv = 1.f / (float)(1 << (2 * (q >> 2)));
          const __half2 bh = __floats2half2_rn(v0 * inv, v1 * inv);
          h2[q] = h2_as_u32(bh);
          cs += (__low2float(bh) + __high2float(bh)) * (1024.f + 2.f * (float)(1 << (2 * (q >> 2))));
        } else {
          h2[q] = h2_as_u32(__floats2half2_rn(v0, v1));
        }
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) out[t] = make_uint4(h2[t], h2[4 + t], h2[8 + t], h2[12 + t]);
      corr[c * kMaxDecodeT + n] = cs;
      if (bad) record_error(ctl, kErrNonFinite, 0x400);
    } else {
      corr[c * kMaxDecodeT + n] = 0.f;
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) xs[c * 32 + n * 4 + t] = out[t];
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  if (warp == 0) build_expert_list(ids, wts, T, L, list, first + L.E, first, ctl);
  __syncthreads();

  const int Fs16 = L.Fs / kTileRows, F16 = L.F / kTileRows;
  const int n_items = Fs16 + (list->n - (L.Fs > 0 ? 1 : 0)) * F16;
  const int my_items = n_items > (int)blockIdx.x ? (n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int quad = warp >> 2, wq = warp & 3, nquads = kGuWarps / 4;
  const int npieces = (nG + kGuPiece - 1) / kGuPiece;
  const int ppw = npieces > wq ? (npieces - 1 - wq) / 4 + 1 : 0;   // pieces per item for this warp
  const int q_items = my_items > quad ? (my_items - 1 - quad) / nquads + 1 : 0;
  const int total = q_items * ppw;           // this warp's (item, piece) sequence
  unsigned char* wst = smem + m.stages + (size_t)warp * spw * m.stage_bytes;
  const size_t LO = kGuPiece * kTileRows * 8, HI = BITS == 3 ? kGuPiece * kTileRows * 4 : 0;
  const size_t hwst = hw_expert_halves(Fmax, T);

  auto issue = [&](int q) {   // sequence index q -> (item li, piece wq + 4*j); whole warp
    const int li = q / ppw, p = wq + 4 * (q % ppw);
    const int it = quad + li * nquads;
    int u, tile;
    gu_item(L, blockIdx.x + it * gridDim.x, Fs16, F16, &u, &tile);
    gu_copy<BITS>(L, list, u, tile, p, wst + (size_t)(q % spw) * m.stage_bytes, ctl);
  };
  for (int q = 0; q < spw && q < total; ++q) issue(q);
  int issued = spw < total ? spw : total;

  int seq = 0;
  for (int li = 0; li < q_items; ++li) {
    float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < ppw; ++j, ++seq) {
      const int s = seq % spw, p = wq + 4 * j;
      cp_async_wait_upto(issued - 1 - seq);   // this piece's group has landed
      __syncwarp();
      {
        const unsigned char* st = wst + (size_t)s * m.stage_bytes;
        const __half* scg = reinterpret_cast<const __half*>(st + 2 * (LO + HI));
        const __half* scu = scg + kGuPiece * kTileRows;
        const int g0 = kGuPiece * p, np = min(kGuPiece, nG - g0);
#pragma unroll 4
        for (int c = 0; c < np; ++c) {
          const uint4 xf = xs[(g0 + c) * 32 + lane];
          const uint32_t b[4] = {xf.x, xf.y, xf.z, xf.w};
          if (BITS == 2) {
            const float2 cr = *reinterpret_cast<const float2*>(corr + (g0 + c) * kMaxDecodeT + 2 * (lane & 3));
            group_mma_2b_offset(st, scg, c, b, cr, accg);
            group_mma_2b_offset(st + LO + HI, scu, c, b, cr, accu);
          } else {
            group_mma<BITS>(st, st + LO, scg, c, b, accg);
            group_mma<BITS>(st + LO + HI, st + 2 * LO + HI, scu, c, b, accu);
          }
        }
      }
      __syncwarp();
      // the stage is free again: refill it with the piece spw steps ahead
      if (issued < total) {
        issue(issued);
        ++issued;
      }
    }
    float* pb = part + ((size_t)(quad * 2 + (li & 1)) * 4) * 32 * 8;
    *reinterpret_cast<float4*>(pb + (wq * 32 + lane) * 8) = make_float4(accg[0], accg[1], accg[2], accg[3]);
    *reinterpret_cast<float4*>(pb + (wq * 32 + lane) * 8 + 4) = make_float4(accu[0], accu[1], accu[2], accu[3]);
    named_bar_sync(1 + quad, 128);
    // warp wq finishes fragment element e = wq of every lane:
    // row g + 8*(e>>1), token 2t + (e&1)
    {
      const int e = wq, g = lane >> 2, t = lane & 3;
      const int n = 2 * t + (e & 1);
      float gv = 0.f, up = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        gv += pb[(w * 32 + lane) * 8 + e];
        up += pb[(w * 32 + lane) * 8 + 4 + e];
      }
      if (n < T) {
        const int it = quad + li * nquads;
        int u, tile;
        gu_item(L, blockIdx.x + it * gridDim.x, Fs16, F16, &u, &tile);
        const float hv = gv / (1.f + expf(-gv)) * up * list->w[u][n];
        // the fp16 hidden value: out-of-range values are flagged (always on)
        if (!(fabsf(hv) <= 65504.f)) record_error(ctl, kErrNonFinite, 0x402);
        const int f = tile * kTileRows + g + 8 * (e >> 1);
        const int c = f >> 5, kk = f & 31, mm = kk >> 3, tt = (kk & 7) >> 1, hh = kk & 1;
        hw[(size_t)u * hwst + ((size_t)c * 4 * T + n * 4 + tt) * 8 + mm * 2 + hh] = __float2half_rn(hv);
      }
    }
  }
  cp_async_wait<0>();   // no copy may still be landing in this warp's stages
}

// ------------------------------------------------------------------- down
struct DnSmem {
  size_t bars, list, first, red, stages, total, stage_bytes, w_bytes;
  int spw;
};
__host__ __device__ inline DnSmem dn_smem(int E, int bits, int Fmax, int T, int spw) {
  DnSmem m;
  size_t o = 0;
  m.spw = spw;
  m.bars = o;
  o += (size_t)kDnWarps * spw * sizeof(uint64_t);
  o = (o + 15) & ~size_t(15);
  m.list = o;
  o += sizeof(ExpList);
  o = (o + 15) & ~size_t(15);
  m.first = o;
  o += 2 * (size_t)E * sizeof(int);   // first-occurrence scratch, slot table
  o = (o + 15) & ~size_t(15);
  m.red = o;
  o += kDnWarps * 32 * 4 * sizeof(float);
  o = (o + 127) & ~size_t(127);
  m.stages = o;
  const int nGF = Fmax / kGroup;
  m.w_bytes = (size_t)nGF * kTileRows * group_bytes(bits) + (size_t)nGF * kTileRows * 2;
  m.stage_bytes = m.w_bytes + hw_expert_halves(Fmax, T) * 2;
  o += (size_t)kDnWarps * spw * m.stage_bytes;
  m.total = o;
  return m;
}

// One CTA per 16-row tile of the output; warp w sums experts w, w+16, ...
// through its private stages.  A stage holds expert u's Wd tile (requested as
// soon as the routing is known, before this grid waits for the gate/up kernel)
// and its hidden vector hw_u (requested after the wait): the stage barrier
// expects two arrivals.  The warps' partial sums are added in a fixed order:
// deterministic, no atomics.
template <int BITS>
__global__ void __launch_bounds__(kDnWarps * 32, 1)
    decode_dn_kernel(LayerDev L, const uint16_t* __restrict__ x, int T,
                     const int32_t* __restrict__ ids, const float* __restrict__ wts,
                     const __half* __restrict__ hw, uint16_t* __restrict__ y, int Fmax,
                     uint32_t flags, Control* ctl, int spw) {
  extern __shared__ __align__(128) unsigned char smem[];
  const DnSmem m = dn_smem(L.E, BITS, Fmax, T, spw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + m.bars);
  ExpList* list = reinterpret_cast<ExpList*>(smem + m.list);
  int* first = reinterpret_cast<int*>(smem + m.first);
  float* red = reinterpret_cast<float*>(smem + m.red);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = L.d, tau = blockIdx.x;
  if (tid == 0) {
    for (int s = 0; s < kDnWarps * spw; ++s) mbar_init(&bars[s], 2);
    fence_barrier_init();
  }
  expert_list_prologue(L, list, first + L.E, first, ctl);
  __syncthreads();
  // The routing lists were written two launches back (the router): readable
  // before this grid waits on decode_gu.
  if (warp == 0) build_expert_list(ids, wts, T, L, list, first + L.E, first, ctl);
  __syncthreads();
  const int n_exp = list->n;
  const size_t hwst = hw_expert_halves(Fmax, T);
  const int mine = n_exp > warp ? (n_exp - 1 - warp) / kDnWarps + 1 : 0;
  unsigned char* wst = smem + m.stages + (size_t)warp * spw * m.stage_bytes;
  uint64_t* wbar = bars + warp * spw;

  auto issue_w = [&](int j) {
    const int u = warp + j * kDnWarps, s = j % spw;
    const ExpSrc src = expert_src(L, list, u, ctl);
    const int nGF = src.F / kGroup;
    const size_t tcb = (size_t)nGF * kTileRows * group_bytes(BITS);
    const size_t tsb = (size_t)nGF * kTileRows * 2;
    const long long mcb = mat_codes_bytes(src.F, d, BITS);
    unsigned char* st = wst + (size_t)s * m.stage_bytes;
    mbar_arrive_expect_tx(&wbar[s], (uint32_t)(tcb + tsb));
    bulk_g2s(st, src.codes + 2 * mcb + (long long)tau * tcb, (uint32_t)tcb, &wbar[s]);
    bulk_g2s(st + tcb, src.scales + 2LL * src.F * (d / kGroup) + (long long)tau * kTileRows * nGF,
             (uint32_t)tsb, &wbar[s]);
  };
  auto issue_h = [&](int j) {
    const int u = warp + j * kDnWarps, s = j % spw;
    const int F = list->id[u] < 0 ? L.Fs : L.F;
    const uint32_t hb = (uint32_t)(F * T * 2);
    mbar_arrive_expect_tx(&wbar[s], hb);
    bulk_g2s(wst + (size_t)s * m.stage_bytes + m.w_bytes, hw + (size_t)u * hwst, hb, &wbar[s]);
  };
  const int pre = mine < spw ? mine : spw;
  if (lane == 0)
    for (int j = 0; j < pre; ++j) issue_w(j);
  pdl_wait();   // hidden vectors come from decode_gu
  pdl_launch_dependents();
  if (lane == 0)
    for (int j = 0; j < pre; ++j) issue_h(j);
  int issued = pre;

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < mine; ++j) {
    const int u = warp + j * kDnWarps, s = j % spw;
    if (!mbar_wait(&wbar[s], (j / spw) & 1, ctl, 0x501)) break;   // no barrier inside the loop
    const int F = list->id[u] < 0 ? L.Fs : L.F;
    const int nGF = F / kGroup;
    const size_t tcb = (size_t)nGF * kTileRows * group_bytes(BITS);
    const unsigned char* st = wst + (size_t)s * m.stage_bytes;
    const __half* sc = reinterpret_cast<const __half*>(st + tcb);
    const uint4* hws = reinterpret_cast<const uint4*>(st + m.w_bytes);
#pragma unroll 4
    for (int c = 0; c < nGF; ++c) {
      uint4 bf = make_uint4(0, 0, 0, 0);
      if (lane < 4 * T) bf = hws[c * 4 * T + lane];
      const uint32_t b[4] = {bf.x, bf.y, bf.z, bf.w};
      group_mma<BITS>(st, st + nGF * kTileRows * 8, sc, c, b, acc);
    }
    __syncwarp();
    if (issued < mine) {
      if (lane == 0) {
        fence_proxy_async_smem();
        issue_w(issued);
        issue_h(issued);
      }
      ++issued;
    }
  }
  if (lane == 0)
    for (int j = issued > spw ? issued - spw : 0; j < issued; ++j)
      mbar_wait(&wbar[j % spw], (j / spw) & 1, ctl, 0x502);
  *reinterpret_cast<float4*>(red + (warp * 32 + lane) * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  __syncthreads();
  if (tid < 128) {
    const int r = tid >> 3, n = tid & 7;
    if (n < T) {
      const int l = (r & 7) * 4 + (n >> 1), idx = (r >> 3) * 2 + (n & 1);
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kDnWarps; ++w) v += red[(w * 32 + l) * 4 + idx];
      const int i = tau * kTileRows + r;
      if (flags & MOE_F_RESIDUAL) v += bf16_bits_to_float(x[(size_t)n * d + i]);
      __nv_bfloat16 bv = __float2bfloat16_rn(v);
      y[(size_t)n * d + i] = *reinterpret_cast<uint16_t*>(&bv);
    }
  }
}

// -------------------------------------------------------------- launcher
constexpr size_t kGuSmemBudget = 215 * 1024;
constexpr size_t kDnSmemBudget = 215 * 1024;

// The stage counts above aim at the budgets; with one stage per warp a launch
// may go up to the sm_100 opt-in maximum of shared memory per block (232448
// bytes), less a margin for the kernels' static shared variables.
constexpr size_t kSmemPerBlockMax = 232448 - 256;

// Whether a T-token window of this layer fits the decode kernels: one stage per
// warp must hold a whole expert's Wd tile and hidden vectors (16 warps), and
// the gate/up kernel its token copies.  Wider experts take the prefill path.
bool decode_fits(int d, int E, int Fmax, int bits, int T) {
  if (d <= 0 || E <= 0 || Fmax <= 0 || T < 1 || T > kMaxDecodeT || (bits != 2 && bits != 3))
    return false;
  return gu_smem(d, E, bits, 1).total <= kSmemPerBlockMax &&
         dn_smem(E, bits, Fmax, T, 1).total <= kSmemPerBlockMax;
}

template <int BITS>
static cudaError_t launch_decode_bits(const LayerDev& L, const uint16_t* x, int T,
                                      const int32_t* ids, const float* w, uint16_t* y,
                                      uint32_t flags, char* ws, const WsLayout& lay,
                                      cudaStream_t st) {
  Control* ctl = reinterpret_cast<Control*>(ws + lay.ctl);
  __half* hw = reinterpret_cast<__half*>(ws + lay.hw);
  const int Fmax = L.F > L.Fs ? L.F : L.Fs;
  const int max_exp = (T * L.k < L.E ? T * L.k : L.E) + (L.Fs > 0 ? 1 : 0);
  // gate/up: private stages per warp, as many as fit (1..4)
  int spw = 4;
  GuSmem gm = gu_smem(L.d, L.E, BITS, spw);
  while (gm.total > kGuSmemBudget && spw > 1) gm = gu_smem(L.d, L.E, BITS, --spw);
  const int max_items = L.Fs / kTileRows + (max_exp - (L.Fs > 0 ? 1 : 0)) * (L.F / kTileRows);
  int grid_gu = sm_count();
  if (grid_gu > max_items) grid_gu = max_items;
  cudaError_t e = cudaFuncSetAttribute(decode_gu_kernel<BITS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gm.total);
  if (e != cudaSuccess) return e;
  e = launch_pdl(decode_gu_kernel<BITS>, dim3(grid_gu), dim3(kGuWarps * 32), gm.total, st, L, x, T,
                 ids, w, hw, Fmax, flags, ctl, spw);
  if (e != cudaSuccess) return e;
  // down: enough private stages per warp to hold all its experts when they fit
  int dspw = (max_exp + kDnWarps - 1) / kDnWarps;
  if (dspw > 6) dspw = 6;
  DnSmem dm = dn_smem(L.E, BITS, Fmax, T, dspw);
  while (dm.total > kDnSmemBudget && dspw > 1) dm = dn_smem(L.E, BITS, Fmax, T, --dspw);
  e = cudaFuncSetAttribute(decode_dn_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)dm.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_dn_kernel<BITS>, dim3(L.d / kTileRows), dim3(kDnWarps * 32), dm.total,
                    st, L, x, T, ids, w, static_cast<const __half*>(hw), y, Fmax, flags, ctl, dspw);
}

cudaError_t launch_decode(const LayerDev& L, const uint16_t* x, int T, const int32_t* ids,
                          const float* w, uint16_t* y, uint32_t flags, char* ws, const WsLayout& lay,
                          cudaStream_t st) {
  if (L.bits == 2) return launch_decode_bits<2>(L, x, T, ids, w, y, flags, ws, lay, st);
  return launch_decode_bits<3>(L, x, T, ids, w, y, flags, ws, lay, st);
}

size_t decode_hw_bytes(const LayerDev& L, int T) {
  const int Fmax = L.F > L.Fs ? L.F : L.Fs;
  const int max_exp = (T * L.k < L.E ? T * L.k : L.E) + (L.Fs > 0 ? 1 : 0);
  return (size_t)max_exp * hw_expert_halves(Fmax, T) * sizeof(__half);
}

}  // namespace moe
