// decode.cu -- decode / verify-window expert step (T <= 8 tokens).
//
// "Checking several tokens costs little more than writing one: the common
// weights are read once and only the experts the extra tokens route to add
// work" ("Why Strata is fast on low-VRAM GPUs", section "guess first, then
// check").  So the window's selected experts are deduplicated and every
// selected expert's packed weights are streamed from HBM exactly once per call.
//
// Split-K over the expert's hidden dimension.  A work unit is one 32-row slice
// s of one expert u: rows 32s..32s+31 of Wg and Wu (two packed 16-row tiles
// each) and the matching 32-column group of Wd (one quantisation group of every
// output row).  A CTA computes the slice's gate/up products, applies SwiGLU
// and the routing weight, and multiplies the 32 hidden values of each token
// with its Wd columns: the hidden vector never leaves the SM.  Each CTA adds
// its units' contributions to all d outputs in registers and writes one fp32
// partial sum per token and output; a small combine kernel adds the CTAs'
// partial sums in CTA order (deterministic, no atomics), adds the residual and
// rounds once to bf16.
//
// One unit arrives as three equal pieces of d*(code bytes per group + 2) bytes
// each: the Wg slice and the Wu slice (two bulk copies each: codes and scales,
// contiguous in the packed layout) and the Wd group column (strided across the
// output-row tiles: one 4-D TMA load per plane).  Pieces stream through a ring
// of shared-memory slots with one mbarrier each; one thread issues them in the
// order they are consumed.
//
// Kernels of a window, chained with programmatic dependent launch (PDL):
//   router (router.cu) -> decode_expert_kernel -> decode_combine_kernel.
// decode_expert_kernel selects the window's top-k itself from the router's
// fp32 logits (every CTA, redundantly: no extra launch and no serial tail)
// and deduplicates the selections; the shared expert's units are requested
// before the kernel waits for the router, since they do not depend on it.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"
#include "select.cuh"
#include "tc.cuh"

namespace moe {

constexpr int kMaxExp = kMaxDecodeT * 16 + 1;   // window entries + shared
constexpr int kDecWarps = 16;

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
#pragma unroll 1
  for (int e = threadIdx.x; e < L.E; e += blockDim.x) {
    int sl = L.slot[e];
    if (sl < 0 || sl >= L.E) {
      record_error(ctl, kErrRange, 0x301);
      sl = 0;
    }
    slot_s[e] = sl;
    first[e] = 0x7FFFFFFF;
  }
#pragma unroll 1
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


// ------------------------------------------------------------- tensor maps
// The down projection's 32-column group s of every 16-row output tile, for
// one slot: 4-D views of the packed Wd bytes (see dec_maps()).
struct alignas(64) DecMaps {
  CUtensorMap lo, hi, sc;      // routed experts (slot dimension = n_experts)
  CUtensorMap slo, shi, ssc;   // shared expert (slot dimension = 1)
};

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------ smem layout
// piece: bytes of one Wg slice, one Wu slice or one Wd group column (equal).
__host__ __device__ inline uint32_t dec_piece_bytes(int d, int bits) {
  return (uint32_t)d * (uint32_t)(group_bytes(bits) + 2);
}
struct DecSmem {
  size_t bars, list, first, sel, xs, corr, part, hfrag, slots, total;
  size_t slot;   // slot stride (a piece, rounded up to 128 bytes)
};
__host__ __device__ inline DecSmem dec_smem(int d, int E, int bits, int nslots) {
  DecSmem m;
  const int nG = d / kGroup;
  size_t o = 0;
  m.bars = o;
  o += (size_t)nslots * sizeof(uint64_t);
  o = (o + 15) & ~size_t(15);
  m.list = o;
  o += sizeof(ExpList);
  o = (o + 15) & ~size_t(15);
  m.first = o;
  o += 2 * (size_t)E * sizeof(int);   // first-occurrence scratch, slot table
  o = (o + 15) & ~size_t(15);
  m.sel = o;                                       // ids int32 [T][k], weights fp32 [T][k]
  o += 2 * (size_t)kMaxDecodeT * 16 * 4;
  o = (o + 127) & ~size_t(127);
  m.xs = o;                                        // B fragments of the tokens, per group
  o += (size_t)nG * 32 * 16;
  m.corr = o;                                      // 2-bit offset-form correction [group][token]
  o += (size_t)nG * kMaxDecodeT * sizeof(float);   // (xs and corr: one bulk copy, in this order)
  o = (o + 15) & ~size_t(15);
  m.part = o;                                      // gate/up partial sums [warp][tile][lane][4]
  o += (size_t)kDecWarps * 2 * 32 * 4 * sizeof(float);
  m.hfrag = o;                                     // hidden slice as down B fragments [lane][4]
  o += 32 * 4 * sizeof(uint32_t);
  o = (o + 127) & ~size_t(127);
  m.slots = o;
  m.slot = ((size_t)dec_piece_bytes(d, bits) + 127) & ~size_t(127);
  o += (size_t)nslots * m.slot;
  m.total = o;
  return m;
}

// Source of list position u (the shared expert when id < 0).
struct ExpSrc {
  const uint8_t* codes;
  const uint16_t* scales;
  int F;
  int slot;   // TMA slot coordinate (0 for the shared expert)
  bool shared;
};
__device__ __forceinline__ ExpSrc expert_src(const LayerDev& L, bool shared, int slot) {
  ExpSrc r;
  r.shared = shared;
  if (shared) {
    r.codes = L.scodes;
    r.scales = L.sscales;
    r.F = L.Fs;
    r.slot = 0;
  } else {
    r.codes = L.codes + (long long)slot * L.cbe;
    r.scales = L.scales + (long long)slot * L.nse;
    r.F = L.F;
    r.slot = slot;
  }
  return r;
}

// Request piece `kind` (0 = Wg slice, 1 = Wu slice, 2 = Wd group column) of
// slice s of expert `src` into `dst`; completion on `bar` (one arrival plus the
// piece's bytes).  One thread.
template <int BITS>
__device__ __noinline__ void issue_piece(const DecMaps& maps, const LayerDev& L, const ExpSrc& src,
                                            int s, int kind, unsigned char* dst, uint64_t* bar) {
  const int d = L.d, nG = d / kGroup, gb = group_bytes(BITS);
  mbar_arrive_expect_tx(bar, dec_piece_bytes(d, BITS));
  if (kind < 2) {
    const long long tcb = (long long)nG * kTileRows * gb;   // code bytes of a 16-row tile
    const long long mcb = (long long)src.F * nG * gb;        // code bytes of an F x d matrix
    const long long msc = (long long)src.F * nG;             // scales of an F x d matrix
    bulk_g2s(dst, src.codes + kind * mcb + 2LL * s * tcb, (uint32_t)(2 * tcb), bar);
    bulk_g2s(dst + 2 * tcb, src.scales + kind * msc + 2LL * s * kTileRows * nG,
             (uint32_t)(2 * kTileRows * nG * 2), bar);
  } else {
    const CUtensorMap* lo = src.shared ? &maps.slo : &maps.lo;
    const CUtensorMap* hi = src.shared ? &maps.shi : &maps.hi;
    const CUtensorMap* sc = src.shared ? &maps.ssc : &maps.sc;
    tma_load_4d(dst, lo, 0, s, 0, src.slot, bar);
    if (BITS == 3) tma_load_4d(dst + 8 * d, hi, 0, s, 0, src.slot, bar);
    tma_load_4d(dst + gb * d, sc, 0, s, 0, src.slot, bar);
  }
}

// ------------------------------------------------------------ expert kernel
// One CTA per SM (grid G).  Units in list order (the shared expert's slices
// first, then each routed expert's in first-occurrence order of the window);
// unit n runs on CTA n % G.  NRT: output-row tiles per warp (d / 256, rounded
// up to 8 or 16).
//
// Warp roles inside a unit: gate/up -- warp w takes matrix w / 8 (Wg, Wu) and
// the K-eighth w % 8 of both 16-row tiles of the slice, so each token fragment
// it loads serves two tiles; the eight partial sums of a (matrix, tile) are
// added in warp order.  Down -- warp w takes the output-row tiles w, w+16, ...
// of the Wd group column and keeps their sums in registers across units.
// The tokens' B fragments (and, for 2-bit, the offset-form corrections) come
// precomputed from the router kernel: one bulk copy.
// At most 88 registers per thread, so that a router or combine CTA can stay
// resident beside it (programmatic dependent launch overlaps the kernels).
template <int BITS, int NRT>
__global__ void __maxnreg__(88)
    decode_expert_kernel(const __grid_constant__ DecMaps maps, const __grid_constant__ LayerDev L,
                         const unsigned char* __restrict__ xfrag, int T,
                         const float* __restrict__ logits, const int32_t* __restrict__ ids_in,
                         const float* __restrict__ w_in, int32_t* __restrict__ ids_out,
                         float* __restrict__ w_out, float* __restrict__ partial, uint32_t flags,
                         Control* ctl, int nslots) {
  extern __shared__ __align__(128) unsigned char smem[];
  const DecSmem m = dec_smem(L.d, L.E, BITS, nslots);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + m.bars);
  ExpList* list = reinterpret_cast<ExpList*>(smem + m.list);
  int* first = reinterpret_cast<int*>(smem + m.first);
  int* slot_s = first + L.E;
  int32_t* sel_ids = reinterpret_cast<int32_t*>(smem + m.sel);
  float* sel_w = reinterpret_cast<float*>(sel_ids + kMaxDecodeT * 16);
  const uint4* xs = reinterpret_cast<const uint4*>(smem + m.xs);
  const float* corr = reinterpret_cast<const float*>(smem + m.corr);
  float* part = reinterpret_cast<float*>(smem + m.part);
  __half* hfrag = reinterpret_cast<__half*>(smem + m.hfrag);
  unsigned char* slots = smem + m.slots;
  __shared__ __align__(8) uint64_t xbar;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = L.d, nG = d / kGroup, gb = group_bytes(BITS);
  const int G = gridDim.x;
  const int sh_units = L.Fs / 32, Fu = L.F / 32;
  const long long tcb = (long long)nG * kTileRows * gb;
  auto slot_ptr = [&](int p) { return slots + (size_t)(p % nslots) * m.slot; };

  if (tid == 0) {
    for (int s = 0; s < nslots; ++s) mbar_init(&full[s], 1);
    mbar_init(&xbar, 1);
    fence_barrier_init();
  }
  // the tensor-map descriptors in use into the TMA unit's cache
  if (warp == 1 && lane < 6 && (BITS == 3 || lane % 3 != 1) && (lane < 3 || L.Fs > 0)) {
    const CUtensorMap* mp = &maps.lo + lane;
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(mp)) : "memory");
  }
  expert_list_prologue(L, list, slot_s, first, ctl);
  __syncthreads();

  // The shared expert's first unit does not depend on the routing: request it
  // before waiting for the router.  Until the first unit's slices have landed
  // only one unit is in flight, so that it is not queued behind the whole
  // GPU's requests; then the ring fills up.
  int issued = 0;   // pieces requested (thread 0)
  int cap = 3;      // pieces allowed ahead of the consumer
  if (tid == 0 && sh_units > (int)blockIdx.x) {
    for (int p = 0; p < 3 && p < nslots; ++p) {
      issue_piece<BITS>(maps, L, expert_src(L, true, 0), blockIdx.x, p, slot_ptr(p), &full[p]);
      issued = p + 1;
    }
  }

  pdl_wait();   // router logits (or the given routing) and the token fragments are complete
  pdl_launch_dependents();
  if (tid == 0) {
    const uint32_t xb = (uint32_t)nG * (32 * 16 + kMaxDecodeT * 4);
    mbar_arrive_expect_tx(&xbar, xb);
    bulk_g2s(smem + m.xs, xfrag, xb, &xbar);
  }

  // ---- routing of the window (warps 0..T-1 select from the logits)
  if (logits) {
    if (warp < T) {
      const float* row = logits + (size_t)warp * L.E;
      if (L.E <= 512)
        warp_topk_n<16>(row, L.E, L.k, sel_ids + warp * L.k, sel_w + warp * L.k, ctl, flags & MOE_F_DEBUG);
      else
        warp_topk_n<32>(row, L.E, L.k, sel_ids + warp * L.k, sel_w + warp * L.k, ctl, flags & MOE_F_DEBUG);
    }
  } else {
#pragma unroll 1
    for (int i = tid; i < T * L.k; i += blockDim.x) {
      sel_ids[i] = __ldcg(ids_in + i);
      sel_w[i] = __ldcg(w_in + i);
    }
  }
  __syncthreads();
  if (warp == 0) build_expert_list(sel_ids, sel_w, T, L, list, slot_s, first, ctl);
  __syncthreads();
  if (blockIdx.x == 0 && ids_out) {
    for (int i = tid; i < T * L.k; i += blockDim.x) {
      ids_out[i] = sel_ids[i];
      w_out[i] = sel_w[i];
    }
  }

  const int n_units = sh_units + (list->n - (L.Fs > 0 ? 1 : 0)) * Fu;
  if (blockIdx.x == 0 && tid == 0) ctl->decode_ctas = (uint32_t)(n_units < G ? n_units : G);
  const int my = n_units > (int)blockIdx.x ? (n_units - 1 - (int)blockIdx.x) / G + 1 : 0;
  const int npieces = 3 * my;
  auto unit_src = [&](int j, int* s) {
    const int n = blockIdx.x + j * G;
    if (n < sh_units) {
      *s = n;
      return expert_src(L, true, 0);
    }
    const int u = (L.Fs > 0 ? 1 : 0) + (n - sh_units) / Fu;
    *s = (n - sh_units) % Fu;
    return expert_src(L, false, list->slot[u]);
  };
  auto unit_u = [&](int j) {
    const int n = blockIdx.x + j * G;
    return n < sh_units ? 0 : (L.Fs > 0 ? 1 : 0) + (n - sh_units) / Fu;
  };
  auto refill = [&](int consumed) {   // thread 0: keep the ring full, in consumption order
    const int lim = consumed + (cap < nslots ? cap : nslots);
    while (issued < npieces && issued < lim) {
      int s;
      const ExpSrc src = unit_src(issued / 3, &s);
      issue_piece<BITS>(maps, L, src, s, issued % 3, slot_ptr(issued), &full[issued % nslots]);
      ++issued;
    }
  };
  if (tid == 0) refill(0);
  bool ok = mbar_wait(&xbar, 0, ctl, 0x600);

  float accd[NRT][4];
#pragma unroll
  for (int i = 0; i < NRT; ++i) accd[i][0] = accd[i][1] = accd[i][2] = accd[i][3] = 0.f;
  const int ntiles = d / kTileRows;
  const int mat = warp >> 3, kq = warp & 7;
  const int c0 = kq * nG / 8, c1 = (kq + 1) * nG / 8;
  int j = 0;
  for (; j < my; ++j) {
    const int pg = 3 * j, pu = pg + 1, pd = pg + 2;
    ok = ok && mbar_wait(&full[pg % nslots], (pg / nslots) & 1, ctl, 0x601);
    ok = ok && mbar_wait(&full[pu % nslots], (pu / nslots) & 1, ctl, 0x602);
    if (!__syncthreads_and(ok)) break;
    if (j == 0 && tid == 0) {   // the first unit is here: let the ring fill
      cap = nslots;
      refill(0);
    }
    // gate/up: warp (matrix, K eighth), both tiles of the slice
    {
      const unsigned char* pc = slot_ptr(mat ? pu : pg);
      const __half* sc = reinterpret_cast<const __half*>(pc + 2 * tcb);
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
      for (int c = c0; c < c1; ++c) {
        const uint4 xf = xs[c * 32 + lane];
        const uint32_t b[4] = {xf.x, xf.y, xf.z, xf.w};
        if (BITS == 2) {
          const float2 cr = *reinterpret_cast<const float2*>(corr + c * kMaxDecodeT + 2 * (lane & 3));
          group_mma_2b_offset(pc, sc, c, b, cr, a0);
          group_mma_2b_offset(pc + tcb, sc + kTileRows * nG, c, b, cr, a1);
        } else {
          group_mma<BITS>(pc, pc + nG * kTileRows * 8, sc, c, b, a0);
          group_mma<BITS>(pc + tcb, pc + tcb + nG * kTileRows * 8, sc + kTileRows * nG, c, b, a1);
        }
      }
      float4* pw = reinterpret_cast<float4*>(part) + (warp * 2) * 32 + lane;
      pw[0] = make_float4(a0[0], a0[1], a0[2], a0[3]);
      pw[32] = make_float4(a1[0], a1[1], a1[2], a1[3]);
    }
    __syncthreads();
    if (tid == 0) {   // the Wg and Wu slots are free
      fence_proxy_async_smem();
      refill(pg + 2);
    }
    // SwiGLU and routing weight: one (row, token) of the slice per thread
    if (tid < 256) {
      const int htl = tid >> 7, ln = (tid >> 2) & 31, e = tid & 3;
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        gs += part[((q * 2 + htl) * 32 + ln) * 4 + e];
        us += part[(((8 + q) * 2 + htl) * 32 + ln) * 4 + e];
      }
      const int row = (ln >> 2) + 8 * (e >> 1) + 16 * htl;   // hidden unit within the slice
      const int n = 2 * (ln & 3) + (e & 1);                   // token
      float h = 0.f;
      if (n < T) h = gs / (1.f + expf(-gs)) * us * list->w[unit_u(j)][n];
      if (!(fabsf(h) <= 65504.f)) record_error(ctl, kErrNonFinite, 0x603);
      // down-projection B fragment: k = row, column = token; 2-bit offset
      // form: the value divided by 4^(k / 8)
      if (BITS == 2) h *= 1.f / (float)(1 << (2 * (row >> 3)));
      const int tp = (row & 7) >> 1, jj = row >> 3, hh = row & 1;
      hfrag[((n * 4 + tp) * 4 + jj) * 2 + hh] = __float2half_rn(h);
    }
    ok = mbar_wait(&full[pd % nslots], (pd / nslots) & 1, ctl, 0x604);
    if (!__syncthreads_and(ok)) break;
    // down: this warp's output-row tiles, one quantisation group each
    {
      const uint4 hb = reinterpret_cast<const uint4*>(hfrag)[lane];
      const uint32_t b[4] = {hb.x, hb.y, hb.z, hb.w};
      const unsigned char* pp = slot_ptr(pd);
      const __half* dsc = reinterpret_cast<const __half*>(pp + gb * d);
      if (BITS == 2) {
        // offset-form correction of token g: sum over the group of
        // B * (1024 + 2 * 4^m); this lane holds 8 of the 32 values (k = 2t +
        // {0,1} + 8m), the four lanes t of the row group hold all of them
        float cs = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __half2 v = u32_as_h2(b[q]);
          cs += (__low2float(v) + __high2float(v)) * (1024.f + 2.f * (float)(1 << (2 * q)));
        }
        cs += __shfl_xor_sync(0xffffffffu, cs, 1);
        cs += __shfl_xor_sync(0xffffffffu, cs, 2);
        const int t = lane & 3;
        const float2 cr = make_float2(__shfl_sync(0xffffffffu, cs, 8 * t),
                                      __shfl_sync(0xffffffffu, cs, 8 * t + 4));
#pragma unroll
        for (int i = 0; i < NRT; ++i) {
          const int r = warp + kDecWarps * i;
          if (r < ntiles) group_mma_2b_offset(pp + r * 128, dsc + r * kTileRows, 0, b, cr, accd[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < NRT; ++i) {
          const int r = warp + kDecWarps * i;
          if (r < ntiles)
            group_mma<BITS>(pp + r * 128, pp + 8 * d + r * 64, dsc + r * kTileRows, 0, b, accd[i]);
        }
      }
    }
    __syncthreads();
    if (tid == 0) {
      fence_proxy_async_smem();
      refill(pg + 3);   // the Wd slot is free
    }
  }
  if (tid == 0) {
    // a wait ran out: let every requested copy land before the CTA exits
    if (j < my)
      for (int p = 3 * j; p < issued; ++p) mbar_wait(&full[p % nslots], (p / nslots) & 1, ctl, 0x605);
    if (!ok) mbar_wait(&xbar, 0, ctl, 0x606);
  }
  // this CTA's partial sums: lane (g, t) of tile r holds rows g, g+8 and tokens 2t, 2t+1
  if (my > 0) {
    const int g = lane >> 2, t = lane & 3;
    float* p0 = partial + ((size_t)blockIdx.x * T + 2 * t) * d + warp * kTileRows + g;
    float* p1 = p0 + d;
    const bool w0 = 2 * t < T, w1 = 2 * t + 1 < T;
#pragma unroll
    for (int i = 0; i < NRT; ++i) {
      if (warp + kDecWarps * i >= ntiles) break;
      const int o = i * kDecWarps * kTileRows;
      if (w0) {
        p0[o] = accd[i][0];
        p0[o + 8] = accd[i][2];
      }
      if (w1) {
        p1[o] = accd[i][1];
        p1[o + 8] = accd[i][3];
      }
    }
  }
}

// ----------------------------------------------------------- combine kernel
// y[n][row] = sum over the expert CTAs c (ascending) of partial[c][n][row]
// (+ x[n][row] with MOE_F_RESIDUAL), rounded once to bf16.  A CTA covers 8
// output rows; its threads split the CTAs into CS strided subsets, and the
// subsets' sums are added in subset order: a fixed order, independent of
// scheduling.
constexpr int kCombRows = 8;
constexpr int kCombThreads = 256;
__global__ void __launch_bounds__(kCombThreads) decode_combine_kernel(
    const float* __restrict__ partial, const uint16_t* __restrict__ x, uint16_t* __restrict__ y,
    int T, int d, uint32_t flags, const Control* ctl) {
  __shared__ float4 red[kCombThreads / 2 * 2];
  // The next kernel of a window chain (the router of the next layer) reads
  // nothing this grid or the expert grid writes before it waits itself.
  pdl_launch_dependents();
  pdl_wait();
  const int nc = (int)*reinterpret_cast<const volatile uint32_t*>(&ctl->decode_ctas);
  const int row0 = blockIdx.x * kCombRows;
  const int CS = (kCombThreads / 2) / T;
  const int tid = threadIdx.x, q = tid & 1, n = (tid >> 1) % T, cs = (tid >> 1) / T;
  if (cs < CS) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    const float* p = partial + (size_t)n * d + row0 + 4 * q;
    const size_t stride = (size_t)T * d;
#pragma unroll 4
    for (int c = cs; c < nc; c += CS) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(p + (size_t)c * stride));
      a.x += v.x;
      a.y += v.y;
      a.z += v.z;
      a.w += v.w;
    }
    red[(cs * T + n) * 2 + q] = a;
  }
  __syncthreads();
  if (tid < kCombRows * T) {
    const int nn = tid / kCombRows, r = tid % kCombRows;
    float v = 0.f;
    for (int c = 0; c < CS; ++c) {
      const float4 a = red[(c * T + nn) * 2 + (r >> 2)];
      v += (r & 3) == 0 ? a.x : (r & 3) == 1 ? a.y : (r & 3) == 2 ? a.z : a.w;
    }
    const size_t i = (size_t)nn * d + row0 + r;
    if (flags & MOE_F_RESIDUAL) v += bf16_bits_to_float(x[i]);
    __nv_bfloat16 bv = __float2bfloat16_rn(v);
    y[i] = *reinterpret_cast<uint16_t*>(&bv);
  }
}

// -------------------------------------------------------------- launcher
// The stage ring takes what is left of 216 KB after the fixed regions (the
// SM's 228 KB then still holds a combine or router CTA beside it, for the
// programmatic overlap); at least two slots (a unit's Wg and Wu slices are
// consumed together), at most eight.
constexpr size_t kSmemPerBlockMax = 216 * 1024;
constexpr int kMaxSlots = 8;

static int dec_nslots(int d, int E, int bits) {
  const DecSmem m0 = dec_smem(d, E, bits, 0);
  if (m0.total >= kSmemPerBlockMax) return 0;
  const size_t n = (kSmemPerBlockMax - m0.total) / m0.slot;
  return n > (size_t)kMaxSlots ? kMaxSlots : (int)n;
}

bool decode_fits(int d, int E, int Fmax, int bits, int T) {
  (void)Fmax;
  if (d <= 0 || E <= 0 || T < 1 || T > kMaxDecodeT || (bits != 2 && bits != 3)) return false;
  return dec_nslots(d, E, bits) >= 2;
}

// ---- tensor maps of the Wd group columns, cached per layer
static PFN_cuTensorMapEncodeTiled_v12000 dec_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

// Wd of an expert with hidden size F in a codes array of `nslot` slots of
// `cbe` bytes: lo plane [slot][tile][group][16 rows x 8 B], hi plane
// [slot][tile][group][16 x 4 B] (3-bit), scales [slot][tile][group][16] fp16.
// Box: group column s of all d/16 tiles of one slot.
static bool dec_encode(CUtensorMap* lo, CUtensorMap* hi, CUtensorMap* sc, const uint8_t* codes,
                       const uint16_t* scales, int d, int F, int bits, int nslot, long long cbe,
                       long long nse) {
  auto fn = dec_encode_fn();
  if (!fn) return false;
  const int gb = group_bytes(bits), nG = d / kGroup, nGF = F / kGroup, ntiles = d / kTileRows;
  const long long mcb = (long long)F * nG * gb;   // code bytes of one F x d matrix
  const cuuint64_t tile_b = (cuuint64_t)nGF * kTileRows * gb;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  {
    cuuint64_t dims[4] = {128, (cuuint64_t)nGF, (cuuint64_t)ntiles, (cuuint64_t)nslot};
    cuuint64_t str[3] = {128, tile_b, (cuuint64_t)cbe};
    cuuint32_t box[4] = {128, 1, (cuuint32_t)ntiles, 1};
    if (fn(lo, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(codes + 2 * mcb), dims, str,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  if (bits == 3) {
    cuuint64_t dims[4] = {64, (cuuint64_t)nGF, (cuuint64_t)ntiles, (cuuint64_t)nslot};
    cuuint64_t str[3] = {64, tile_b, (cuuint64_t)cbe};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)ntiles, 1};
    if (fn(hi, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4,
           const_cast<uint8_t*>(codes + 2 * mcb + (long long)nGF * kTileRows * 8), dims, str, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  } else {
    memset(hi, 0, sizeof(*hi));
  }
  {
    cuuint64_t dims[4] = {16, (cuuint64_t)nGF, (cuuint64_t)ntiles, (cuuint64_t)nslot};
    cuuint64_t str[3] = {32, (cuuint64_t)nGF * 32, (cuuint64_t)nse * 2};
    cuuint32_t box[4] = {16, 1, (cuuint32_t)ntiles, 1};
    if (fn(sc, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4,
           const_cast<uint16_t*>(scales + 2LL * F * nG), dims, str, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

// A small direct-mapped cache of encoded maps, keyed by the layer's pointers
// and shape (encoding costs a few microseconds of host time per map).
struct DecMapEntry {
  const void *codes, *scales, *scodes, *sscales;
  int d, E, F, Fs, bits;
  DecMaps maps;
};
static std::mutex g_map_mu;
static DecMapEntry g_map_cache[1024];

static bool dec_maps(const LayerDev& L, DecMaps* out) {
  const size_t h = ((reinterpret_cast<uintptr_t>(L.codes) >> 8) ^
                    (reinterpret_cast<uintptr_t>(L.scales) >> 4) ^
                    (reinterpret_cast<uintptr_t>(L.scodes) >> 6)) % 1024;
  std::lock_guard<std::mutex> lock(g_map_mu);
  DecMapEntry& e = g_map_cache[h];
  if (e.codes == L.codes && e.scales == L.scales && e.scodes == L.scodes &&
      e.sscales == L.sscales && e.d == L.d && e.E == L.E && e.F == L.F && e.Fs == L.Fs &&
      e.bits == L.bits) {
    *out = e.maps;
    return true;
  }
  DecMaps mp;
  memset(&mp, 0, sizeof(mp));
  if (!dec_encode(&mp.lo, &mp.hi, &mp.sc, L.codes, L.scales, L.d, L.F, L.bits, L.E, L.cbe, L.nse))
    return false;
  if (L.Fs > 0) {
    const long long cbs = 3LL * L.Fs * (L.d / kGroup) * group_bytes(L.bits);
    const long long nss = 3LL * L.Fs * (L.d / kGroup);
    if (!dec_encode(&mp.slo, &mp.shi, &mp.ssc, L.scodes, L.sscales, L.d, L.Fs, L.bits, 1, cbs, nss))
      return false;
  }
  e.codes = L.codes;
  e.scales = L.scales;
  e.scodes = L.scodes;
  e.sscales = L.sscales;
  e.d = L.d;
  e.E = L.E;
  e.F = L.F;
  e.Fs = L.Fs;
  e.bits = L.bits;
  e.maps = mp;
  *out = mp;
  return true;
}

int decode_grid() {
  const int g = sm_count();
  return g < kMaxDecodeCtas ? g : kMaxDecodeCtas;
}

template <int BITS, int NRT>
static cudaError_t launch_expert(const DecMaps& mp, const LayerDev& L, const unsigned char* xfrag, int T,
                                 const float* logits, const int32_t* ids, const float* w,
                                 int32_t* ids_out, float* w_out, float* partial, uint32_t flags,
                                 Control* ctl, int nslots, cudaStream_t st) {
  const DecSmem m = dec_smem(L.d, L.E, BITS, nslots);
  cudaError_t e = cudaFuncSetAttribute(decode_expert_kernel<BITS, NRT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)m.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_expert_kernel<BITS, NRT>, dim3(decode_grid()), dim3(kDecWarps * 32),
                    m.total, st, mp, L, xfrag, T, logits, ids, w, ids_out, w_out, partial, flags, ctl,
                    nslots);
}

cudaError_t launch_decode(const LayerDev& L, const uint16_t* x, int T, const float* logits,
                          const int32_t* ids, const float* w, int32_t* ids_out, float* w_out,
                          uint16_t* y, uint32_t flags, char* ws, const WsLayout& lay,
                          cudaStream_t st) {
  Control* ctl = reinterpret_cast<Control*>(ws + lay.ctl);
  float* partial = reinterpret_cast<float*>(ws + lay.partial);
  const unsigned char* xf = reinterpret_cast<const unsigned char*>(ws + lay.xfrag);
  const int nslots = dec_nslots(L.d, L.E, L.bits);
  if (nslots < 2) return cudaErrorInvalidValue;
  DecMaps mp;
  if (!dec_maps(L, &mp)) return cudaErrorInvalidValue;
  cudaError_t e;
  const bool wide = L.d / kTileRows > kDecWarps * 8;
  if (L.bits == 2)
    e = wide ? launch_expert<2, 16>(mp, L, xf, T, logits, ids, w, ids_out, w_out, partial, flags, ctl, nslots, st)
             : launch_expert<2, 8>(mp, L, xf, T, logits, ids, w, ids_out, w_out, partial, flags, ctl, nslots, st);
  else
    e = wide ? launch_expert<3, 16>(mp, L, xf, T, logits, ids, w, ids_out, w_out, partial, flags, ctl, nslots, st)
             : launch_expert<3, 8>(mp, L, xf, T, logits, ids, w, ids_out, w_out, partial, flags, ctl, nslots, st);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_combine_kernel, dim3(L.d / kCombRows), dim3(kCombThreads), 0, st,
                    static_cast<const float*>(partial), x, y, T, L.d, flags,
                    static_cast<const Control*>(ctl));
}

size_t decode_xfrag_bytes(const LayerDev& L) {
  return (size_t)(L.d / kGroup) * (32 * 16 + kMaxDecodeT * 4);
}

size_t decode_partial_bytes(const LayerDev& L, int T) {
  const int Tn = T < 1 ? 1 : (T > kMaxDecodeT ? kMaxDecodeT : T);
  return (size_t)kMaxDecodeCtas * Tn * L.d * sizeof(float);
}

}  // namespace moe
