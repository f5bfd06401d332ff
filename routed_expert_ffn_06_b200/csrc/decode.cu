// decode.cu -- decode / verify-window expert step (T <= 8 tokens).
//
// "Checking several tokens costs little more than writing one: the common
// weights are read once and only the experts the extra tokens route to add
// work" ("Why Strata is fast on low-VRAM GPUs", section "guess first, then
// check").  So the window's selected experts are deduplicated and every
// selected expert's packed weights are streamed from HBM exactly once per call.
//
// Two kernels, chained with programmatic dependent launch:
//  * decode_gu: work item = (expert u, 16-row tile of Wg/Wu).  A producer warp
//    streams the item's packed tiles into a shared-memory ring with bulk async
//    copies; eight consumer warps split the d/32 groups, dequantise 2/3-bit
//    codes straight into mma.sync A fragments (LOP3 + HFMA2, no shared-memory
//    round trip for the fp16 weights) and multiply them with the window's
//    tokens (B fragments, n = 8 covers T <= 8).  The epilogue reduces the
//    warps, applies SwiGLU and the routing weight, and writes
//    hw[u][f][t] = w_u[t] * silu(g) * up  (fp16, fragment order).
//  * decode_dn: one CTA per 16-row tile of the output.  Its Wd tiles depend
//    only on the routing, so they are fetched before the kernel waits for
//    decode_gu; then the CTA sums over all experts' K in a fixed order (no
//    atomics, deterministic) and writes y (bf16, optional residual).
// The shared expert is expert u = 0 with weight 1 for every token.
#include "internal.h"

namespace moe {

constexpr int kMaxExp = kMaxDecodeT * 16 + 1;   // window entries + shared
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

struct ExpList {
  int n;                       // experts in the list (shared first when present)
  int id[kMaxExp];             // expert id, -1 = shared
  float w[kMaxExp][kMaxDecodeT];
  int uidx[kMaxDecodeT * 16];  // list position of a window entry's expert
};

// Warp 0: deduplicate the window's T*k selections in first-occurrence order.
// Out-of-range ids are dropped and flagged.  first: E ints of scratch.
__device__ void build_expert_list(const int32_t* __restrict__ ids, const float* __restrict__ w,
                                  int T, const LayerDev& L, ExpList* s, int* first, Control* ctl) {
  const int lane = threadIdx.x & 31;
  const int n_ent = T * L.k;
  const int base = L.Fs > 0 ? 1 : 0;
  for (int e = lane; e < L.E; e += 32) first[e] = 0x7FFFFFFF;
  for (int i = lane; i < kMaxExp * kMaxDecodeT; i += 32) (&s->w[0][0])[i] = 0.f;
  __syncwarp();
  int ent[4];
  float entw[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int i = lane + 32 * c;
    ent[c] = -1;
    entw[c] = 0.f;
    if (i < n_ent) {
      int e = ids[i];
      if (e < 0 || e >= L.E) {
        record_error(ctl, kErrRange, 0x300);
        e = -1;
      } else {
        entw[c] = w[i];
        atomicMin(&first[e], i);
      }
      ent[c] = e;
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
// group: acc += scale_row * (A_group . B).  tile: the tile's bytes in shared
// memory, sc: its scales, nG: groups per row.
template <int BITS>
__device__ __forceinline__ void group_mma(const unsigned char* tile, const __half* sc, int nG, int c,
                                          const uint32_t (&b)[4], float (&acc)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint32_t sel = (uint32_t)t | ((uint32_t)(4 + t) << 8);
  const uint2 lo0 = *reinterpret_cast<const uint2*>(tile + (c * 16 + g) * 8);
  const uint2 lo1 = *reinterpret_cast<const uint2*>(tile + (c * 16 + g + 8) * 8);
  uint32_t a0[4], a1[4];
  if (BITS == 2) {
    dq2(lo0, sel, a0);
    dq2(lo1, sel, a1);
  } else {
    const unsigned char* hib = tile + nG * 16 * 8;
    const uint32_t h0 = *reinterpret_cast<const uint32_t*>(hib + (c * 16 + g) * 4);
    const uint32_t h1 = *reinterpret_cast<const uint32_t*>(hib + (c * 16 + g + 8) * 4);
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

// Source of expert u (shared when u == 0 and the layer has one).
struct ExpSrc {
  const uint8_t* codes;
  const uint16_t* scales;
  int F;
};
__device__ __forceinline__ ExpSrc expert_src(const LayerDev& L, const ExpList* s, int u,
                                             Control* ctl) {
  ExpSrc r;
  const int e = s->id[u];
  if (e < 0) {
    r.codes = L.scodes;
    r.scales = L.sscales;
    r.F = L.Fs;
  } else {
    int slot = L.slot[e];
    if (slot < 0 || slot >= L.E) {
      record_error(ctl, kErrRange, 0x301);
      slot = 0;
    }
    r.codes = L.codes + (long long)slot * L.cbe;
    r.scales = L.scales + (long long)slot * L.nse;
    r.F = L.F;
  }
  return r;
}

// ------------------------------------------------------------------ gate/up
struct GuSmem {
  size_t bars, list, first, xs, red, stages, total, item_bytes;
};
__host__ __device__ inline GuSmem gu_smem(int d, int E, int bits, int NS) {
  GuSmem m;
  const int nG = d / kGroup;
  size_t o = 0;
  m.bars = o;
  o += 2 * NS * sizeof(uint64_t);
  o = (o + 15) & ~size_t(15);
  m.list = o;
  o += sizeof(ExpList);
  o = (o + 15) & ~size_t(15);
  m.first = o;
  o += (size_t)E * sizeof(int);
  o = (o + 15) & ~size_t(15);
  m.xs = o;
  o += (size_t)nG * 32 * 16;
  m.red = o;
  o += 2 * kConsumerWarps * 2 * 32 * 4 * sizeof(float);
  o = (o + 127) & ~size_t(127);
  m.stages = o;
  const size_t tcb = (size_t)nG * kTileRows * group_bytes(bits);
  m.item_bytes = 2 * tcb + 2 * (size_t)nG * kTileRows * 2;
  o += (size_t)NS * m.item_bytes;
  m.total = o;
  return m;
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
    decode_gu_kernel(LayerDev L, const uint16_t* __restrict__ x, int T,
                     const int32_t* __restrict__ ids, const float* __restrict__ wts,
                     __half* __restrict__ hw, int Fmax, uint32_t flags, Control* ctl, int NS) {
  extern __shared__ __align__(128) unsigned char smem[];
  const GuSmem m = gu_smem(L.d, L.E, BITS, NS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + m.bars);
  uint64_t* empty = full + NS;
  ExpList* list = reinterpret_cast<ExpList*>(smem + m.list);
  int* first = reinterpret_cast<int*>(smem + m.first);
  uint4* xs = reinterpret_cast<uint4*>(smem + m.xs);
  float* red = reinterpret_cast<float*>(smem + m.red);
  unsigned char* stages = smem + m.stages;
  __shared__ float inv_rms[kMaxDecodeT];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = L.d, nG = d / kGroup;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_barrier_init();
  }
  // ---- tokens -> B fragments (x is an input of the whole block: safe to read
  //      before waiting on the router)
  if (warp < T) {
    float ss = 0.f;
    for (int i = lane; i < d; i += 32) {
      const float v = bf16_bits_to_float(x[(size_t)warp * d + i]);
      ss += v * v;
    }
    ss = warp_sum(ss);
    if (lane == 0) inv_rms[warp] = (flags & MOE_F_PRENORM) ? rsqrtf(ss / (float)d + 1e-6f) : 1.f;
  }
  __syncthreads();
  for (int i = tid; i < nG * 32 * 4; i += kThreads) {
    // i -> (c, lane l, pair m): token n = l / 4, column 32c + 8m + 2(l % 4)
    const int mpair = i & 3, l = (i >> 2) & 31, c = i >> 7;
    const int n = l >> 2, col = 32 * c + 8 * mpair + 2 * (l & 3);
    __half2 v = __float2half2_rn(0.f);
    if (n < T) {
      float v0 = bf16_bits_to_float(x[(size_t)n * d + col]);
      float v1 = bf16_bits_to_float(x[(size_t)n * d + col + 1]);
      if (flags & MOE_F_PRENORM) {
        v0 = __bfloat162float(__float2bfloat16_rn(v0 * inv_rms[n]));
        v1 = __bfloat162float(__float2bfloat16_rn(v1 * inv_rms[n]));
      }
      v = __floats2half2_rn(v0, v1);
    }
    reinterpret_cast<__half2*>(xs)[i] = v;
  }
  pdl_wait();
  pdl_launch_dependents();
  if (warp == 0) build_expert_list(ids, wts, T, L, list, first, ctl);
  __syncthreads();

  const int Fs16 = L.Fs / kTileRows, F16 = L.F / kTileRows;
  const int n_items = Fs16 + (list->n - (L.Fs > 0 ? 1 : 0)) * F16;
  const size_t tcb = (size_t)nG * kTileRows * group_bytes(BITS);
  const size_t tsb = (size_t)nG * kTileRows * 2;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0;; ++it) {
        const int i = blockIdx.x + it * gridDim.x;
        if (i >= n_items) break;
        const int s = it % NS;
        if (it >= NS && !mbar_wait(&empty[s], ((it / NS) - 1) & 1, ctl, 0x400)) break;
        ++issued;
        int u, tile;
        if (i < Fs16) {
          u = 0;
          tile = i;
        } else {
          u = (L.Fs > 0 ? 1 : 0) + (i - Fs16) / F16;
          tile = (i - Fs16) % F16;
        }
        const ExpSrc src = expert_src(L, list, u, ctl);
        unsigned char* st = stages + (size_t)s * m.item_bytes;
        const long long mcb = mat_codes_bytes(src.F, d, BITS);
        const long long msc = (long long)src.F * nG;
        mbar_arrive_expect_tx(&full[s], (uint32_t)m.item_bytes);
        bulk_g2s(st, src.codes + tile * tcb, (uint32_t)tcb, &full[s]);
        bulk_g2s(st + tcb, src.codes + mcb + tile * tcb, (uint32_t)tcb, &full[s]);
        bulk_g2s(st + 2 * tcb, src.scales + (long long)tile * kTileRows * nG, (uint32_t)tsb,
                 &full[s]);
        bulk_g2s(st + 2 * tcb + tsb, src.scales + msc + (long long)tile * kTileRows * nG,
                 (uint32_t)tsb, &full[s]);
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int j = issued > NS ? issued - NS : 0; j < issued; ++j)
        mbar_wait(&full[j % NS], (j / NS) & 1, ctl, 0x403);
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  // A wait that runs out marks the CTA failed: its warps stop reading stages
  // but still take every named barrier, so no warp is left waiting.
  bool ok = true;
  for (int it = 0;; ++it) {
    const int i = blockIdx.x + it * gridDim.x;
    if (i >= n_items) break;
    const int s = it % NS;
    if (ok) ok = mbar_wait(&full[s], (it / NS) & 1, ctl, 0x401);
    const unsigned char* st = stages + (size_t)s * m.item_bytes;
    const __half* scg = reinterpret_cast<const __half*>(st + 2 * tcb);
    const __half* scu = reinterpret_cast<const __half*>(st + 2 * tcb + tsb);
    float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
      for (int c = warp; c < nG; c += kConsumerWarps) {
        const uint4 xf = xs[c * 32 + lane];
        const uint32_t b[4] = {xf.x, xf.y, xf.z, xf.w};
        group_mma<BITS>(st, scg, nG, c, b, accg);
        group_mma<BITS>(st + tcb, scu, nG, c, b, accu);
      }
    }
    __syncwarp();
    if (lane == 0 && ok) mbar_arrive(&empty[s]);
    float* rb = red + (size_t)(it & 1) * kConsumerWarps * 2 * 32 * 4;
    *reinterpret_cast<float4*>(rb + ((warp * 2 + 0) * 32 + lane) * 4) =
        make_float4(accg[0], accg[1], accg[2], accg[3]);
    *reinterpret_cast<float4*>(rb + ((warp * 2 + 1) * 32 + lane) * 4) =
        make_float4(accu[0], accu[1], accu[2], accu[3]);
    named_bar_sync(1, kConsumerWarps * 32);
    if (tid < 128) {
      // (row r, token n) of this 16-row tile
      const int r = tid >> 3, n = tid & 7;
      const int l = (r & 7) * 4 + (n >> 1), idx = (r >> 3) * 2 + (n & 1);
      float g = 0.f, up = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        g += rb[((w * 2 + 0) * 32 + l) * 4 + idx];
        up += rb[((w * 2 + 1) * 32 + l) * 4 + idx];
      }
      int u, tile;
      if (i < Fs16) {
        u = 0;
        tile = i;
      } else {
        u = (L.Fs > 0 ? 1 : 0) + (i - Fs16) / F16;
        tile = (i - Fs16) % F16;
      }
      const float h = g / (1.f + expf(-g)) * up;
      const float hv = h * list->w[u][n];
      if ((flags & MOE_F_DEBUG) && !(fabsf(hv) <= 65504.f)) record_error(ctl, kErrNonFinite, 0x402);
      // hw fragment order: [u][c][lane'][m][2], f = 32c + 8m + 2t' + hh, lane' = n*4 + t'
      const int f = tile * kTileRows + r;
      const int c = f >> 5, kk = f & 31, mm = kk >> 3, tt = (kk & 7) >> 1, hh = kk & 1;
      const size_t off = ((((size_t)u * (Fmax / 32) + c) * 32 + n * 4 + tt) * 4 + mm) * 2 + hh;
      hw[off] = __float2half_rn(hv);
    }
  }
}

// ------------------------------------------------------------------- down
struct DnSmem {
  size_t bars, list, first, red, stages, total, stage_bytes;
};
__host__ __device__ inline DnSmem dn_smem(int E, int bits, int Fmax, int NS) {
  DnSmem m;
  size_t o = 0;
  m.bars = o;
  o += 2 * NS * sizeof(uint64_t);
  o = (o + 15) & ~size_t(15);
  m.list = o;
  o += sizeof(ExpList);
  o = (o + 15) & ~size_t(15);
  m.first = o;
  o += (size_t)E * sizeof(int);
  o = (o + 15) & ~size_t(15);
  m.red = o;
  o += kConsumerWarps * 32 * 4 * sizeof(float);
  o = (o + 127) & ~size_t(127);
  m.stages = o;
  const int nGF = Fmax / kGroup;
  m.stage_bytes = (size_t)nGF * kTileRows * group_bytes(bits) + (size_t)nGF * kTileRows * 2;
  o += (size_t)NS * m.stage_bytes;
  m.total = o;
  return m;
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
    decode_dn_kernel(LayerDev L, const uint16_t* __restrict__ x, int T,
                     const int32_t* __restrict__ ids, const float* __restrict__ wts,
                     const __half* __restrict__ hw, uint16_t* __restrict__ y, int Fmax,
                     uint32_t flags, Control* ctl, int NS) {
  extern __shared__ __align__(128) unsigned char smem[];
  const DnSmem m = dn_smem(L.E, BITS, Fmax, NS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + m.bars);
  uint64_t* empty = full + NS;
  ExpList* list = reinterpret_cast<ExpList*>(smem + m.list);
  int* first = reinterpret_cast<int*>(smem + m.first);
  float* red = reinterpret_cast<float*>(smem + m.red);
  unsigned char* stages = smem + m.stages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = L.d, tau = blockIdx.x;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_barrier_init();
  }
  // The routing lists were written two launches back (the router): readable
  // before this grid waits on decode_gu.
  if (warp == 0) build_expert_list(ids, wts, T, L, list, first, ctl);
  __syncthreads();
  const int n_exp = list->n;

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      int issued = 0;
      for (int u = 0; u < n_exp; ++u) {
        const int s = u % NS;
        if (u >= NS && !mbar_wait(&empty[s], ((u / NS) - 1) & 1, ctl, 0x500)) break;
        const ExpSrc src = expert_src(L, list, u, ctl);
        const int nGF = src.F / kGroup;
        const size_t tcb = (size_t)nGF * kTileRows * group_bytes(BITS);
        const size_t tsb = (size_t)nGF * kTileRows * 2;
        const long long mcb = mat_codes_bytes(src.F, d, BITS);
        unsigned char* st = stages + (size_t)s * m.stage_bytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(tcb + tsb));
        bulk_g2s(st, src.codes + 2 * mcb + (long long)tau * tcb, (uint32_t)tcb, &full[s]);
        bulk_g2s(st + tcb, src.scales + 2LL * src.F * (d / kGroup) + (long long)tau * kTileRows * nGF,
                 (uint32_t)tsb, &full[s]);
        ++issued;
      }
      for (int j = issued > NS ? issued - NS : 0; j < issued; ++j)
        mbar_wait(&full[j % NS], (j / NS) & 1, ctl, 0x502);
    }
    pdl_wait();
    pdl_launch_dependents();
    return;
  }
  pdl_wait();   // hw comes from decode_gu
  pdl_launch_dependents();
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int u = warp; u < n_exp; u += kConsumerWarps) {
    const int s = u % NS;
    if (!mbar_wait(&full[s], (u / NS) & 1, ctl, 0x501)) break;   // no barrier inside the loop
    const int F = list->id[u] < 0 ? L.Fs : L.F;
    const int nGF = F / kGroup;
    const size_t tcb = (size_t)nGF * kTileRows * group_bytes(BITS);
    const unsigned char* st = stages + (size_t)s * m.stage_bytes;
    const __half* sc = reinterpret_cast<const __half*>(st + tcb);
    const uint4* hwu = reinterpret_cast<const uint4*>(hw + (size_t)u * Fmax * 8);
    for (int c = 0; c < nGF; ++c) {
      const uint4 bf = hwu[c * 32 + lane];
      const uint32_t b[4] = {bf.x, bf.y, bf.z, bf.w};
      group_mma<BITS>(st, sc, nGF, c, b, acc);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  *reinterpret_cast<float4*>(red + (warp * 32 + lane) * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  named_bar_sync(1, kConsumerWarps * 32);
  if (tid < 128) {
    const int r = tid >> 3, n = tid & 7;
    if (n < T) {
      const int l = (r & 7) * 4 + (n >> 1), idx = (r >> 3) * 2 + (n & 1);
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) v += red[(w * 32 + l) * 4 + idx];
      const int i = tau * kTileRows + r;
      if (flags & MOE_F_RESIDUAL) v += bf16_bits_to_float(x[(size_t)n * d + i]);
      __nv_bfloat16 bv = __float2bfloat16_rn(v);
      y[(size_t)n * d + i] = *reinterpret_cast<uint16_t*>(&bv);
    }
  }
}

// -------------------------------------------------------------- launcher
constexpr size_t kGuSmemBudget = 200 * 1024;

template <int BITS>
static cudaError_t launch_decode_bits(const LayerDev& L, const uint16_t* x, int T,
                                      const int32_t* ids, const float* w, uint16_t* y,
                                      uint32_t flags, char* ws, const WsLayout& lay,
                                      cudaStream_t st) {
  Control* ctl = reinterpret_cast<Control*>(ws + lay.ctl);
  __half* hw = reinterpret_cast<__half*>(ws + lay.hw);
  const int Fmax = L.F > L.Fs ? L.F : L.Fs;
  const int max_exp = (T * L.k < L.E ? T * L.k : L.E) + (L.Fs > 0 ? 1 : 0);
  // gate/up
  // as many ring stages as fit next to the fixed parts (2..6)
  const GuSmem g0 = gu_smem(L.d, L.E, BITS, 0);
  int NSg = (int)((kGuSmemBudget - g0.total) / g0.item_bytes);
  NSg = NSg < 2 ? 2 : (NSg > 6 ? 6 : NSg);
  const GuSmem gm = gu_smem(L.d, L.E, BITS, NSg);
  const int max_items = L.Fs / kTileRows + (max_exp - (L.Fs > 0 ? 1 : 0)) * (L.F / kTileRows);
  int grid_gu = sm_count();
  if (grid_gu > max_items) grid_gu = max_items;
  cudaError_t e = cudaFuncSetAttribute(decode_gu_kernel<BITS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gm.total);
  if (e != cudaSuccess) return e;
  e = launch_pdl(decode_gu_kernel<BITS>, dim3(grid_gu), dim3(kThreads), gm.total, st, L, x, T, ids,
                 w, hw, Fmax, flags, ctl, NSg);
  if (e != cudaSuccess) return e;
  // down
  int NSd = max_exp < 48 ? max_exp : 48;
  DnSmem dm = dn_smem(L.E, BITS, Fmax, NSd);
  while (dm.total > 200 * 1024 && NSd > 2) {
    --NSd;
    dm = dn_smem(L.E, BITS, Fmax, NSd);
  }
  e = cudaFuncSetAttribute(decode_dn_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)dm.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_dn_kernel<BITS>, dim3(L.d / kTileRows), dim3(kThreads), dm.total, st, L,
                    x, T, ids, w, static_cast<const __half*>(hw), y, Fmax, flags, ctl, NSd);
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
  return (size_t)max_exp * Fmax * 8 * sizeof(__half);
}

}  // namespace moe
