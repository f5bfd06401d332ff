// adapt.cu -- adaptive frequency-ordered slot layout.
//
// The pages' expert cache starts from a popularity ranking and then follows
// the session: it keeps counting the routing, with exponential decay, and
// periodically swaps new hot experts in and cold ones out, a bounded number
// per round ("Strata: Run a 125B Model on a 12 GB GPU with MoE Expert Hot
// Cache", section "How It Works": adaptive eviction with exponential decay;
// "Strata illustrated", section on the expert cache: the adaptive tier, a
// window of --adapt-every rounds, at most 96 swaps per 4 rounds).  Here every
// expert is resident in HBM, so the cache becomes the slot order itself: the
// hottest experts are moved to the lowest, contiguous slots.
//
// Counting happens in the selection (route_counts, one count per pick).  One
// call of moe_adapt_layout:
//  1. adapt_plan_kernel (one CTA): ranks the experts by count (descending,
//     ties to the lower expert index); walks the ranks and, while under the
//     swap budget, swaps the expert of rank r into slot r; writes the new
//     expert -> slot table and the list of moved slots; decays the counts.
//  2. adapt_copy_kernel<true>: the packed bytes (codes and scales) of every
//     moved slot into the workspace's staging area;
//  3. adapt_copy_kernel<false>: from the staging area into their new slots.
// The kernels run in stream order after whatever used the layer before and
// are launched without programmatic overlap, so no kernel reads the layer
// while it is rewritten.
#include "internal.h"

namespace moe {

constexpr int kPlanThreads = 1024;

// Workspace: [control block][n_moves int32, pad][moves: (from, to) int32
// pairs][staging].
struct AdaptWs {
  size_t n_moves, moves, staging, total;
};
static AdaptWs adapt_ws(const LayerDev& L, int max_swaps) {
  AdaptWs w;
  const size_t per = (size_t)L.cbe + (size_t)L.nse * 2;   // one slot's codes and scales
  w.n_moves = sizeof(Control);
  w.moves = w.n_moves + 256;
  w.staging = (w.moves + (size_t)2 * max_swaps * 2 * sizeof(int32_t) + 255) & ~size_t(255);
  w.total = w.staging + (size_t)2 * max_swaps * ((per + 255) & ~size_t(255));
  return w;
}

__global__ void __launch_bounds__(kPlanThreads) adapt_plan_kernel(
    const LayerDev L, int32_t* __restrict__ slot_table, float* __restrict__ counts, float decay,
    int max_swaps, int32_t* __restrict__ n_moves, int32_t* __restrict__ moves,
    int32_t* __restrict__ swaps_done, Control* ctl) {
  __shared__ float c[1024];
  __shared__ int order[1024];
  __shared__ int slot[1024];         // expert -> slot (evolving)
  __shared__ int at[1024];           // slot -> expert (evolving)
  __shared__ int old_slot[1024];
  __shared__ int seen[1024];
  const int E = L.E, tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) seen[e] = 0;
  __syncthreads();
  // the slot table must be a permutation of 0..E-1: otherwise nothing moves
  bool bad = false;
  for (int e = tid; e < E; e += blockDim.x) {
    c[e] = counts[e];
    const int s = slot_table[e];
    slot[e] = s;
    old_slot[e] = s;
    if (s < 0 || s >= E)
      bad = true;
    else
      atomicAdd(&seen[s], 1);
  }
  __syncthreads();
  for (int p = tid; p < E; p += blockDim.x) bad |= seen[p] != 1;
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      *n_moves = 0;
      if (swaps_done) *swaps_done = 0;
      record_error(ctl, kErrRange, 0x700);
    }
    return;
  }
  for (int e = tid; e < E; e += blockDim.x) at[slot[e]] = e;
  // rank of expert e: experts with a larger count, or an equal count and a
  // lower index, come first
  for (int e = tid; e < E; e += blockDim.x) {
    const float ce = c[e];
    int r = 0;
    for (int f = 0; f < E; ++f) r += (c[f] > ce) || (c[f] == ce && f < e);
    order[r] = e;
  }
  __syncthreads();
  if (tid == 0) {
    int nsw = 0;
    for (int r = 0; r < E && nsw < max_swaps; ++r) {
      const int e = order[r], s = slot[e];
      if (s == r) continue;
      const int other = at[r];   // the expert now in slot r moves to e's slot
      slot[e] = r;
      at[r] = e;
      slot[other] = s;
      at[s] = other;
      ++nsw;
    }
    // moved slots: the expert now at slot p came from old_slot[at[p]]
    int nm = 0;
    for (int p = 0; p < E; ++p) {
      const int q = old_slot[at[p]];
      if (q != p) {
        moves[2 * nm] = q;
        moves[2 * nm + 1] = p;
        ++nm;
      }
    }
    *n_moves = nm;
    if (swaps_done) *swaps_done = nsw;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    slot_table[e] = slot[e];
    counts[e] = c[e] * decay;
  }
}

// Copy the moved slots' bytes (codes, then scales) to or from the staging area.
// Grid-stride over (move, 16-byte chunk).
template <bool kGather>
__global__ void __launch_bounds__(256) adapt_copy_kernel(const LayerDev L,
                                                         const int32_t* __restrict__ n_moves,
                                                         const int32_t* __restrict__ moves,
                                                         unsigned char* __restrict__ staging,
                                                         size_t staging_stride) {
  const int nm = *n_moves;
  const size_t cb = (size_t)L.cbe / 16, sb = (size_t)L.nse * 2 / 16, per = cb + sb;
  uint8_t* codes = const_cast<uint8_t*>(L.codes);
  uint8_t* scales = reinterpret_cast<uint8_t*>(const_cast<uint16_t*>(L.scales));
  const size_t total = (size_t)nm * per;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(i / per);
    const size_t j = i % per;
    const int slot = moves[2 * m + (kGather ? 0 : 1)];
    uint4* dev = j < cb ? reinterpret_cast<uint4*>(codes + (size_t)slot * L.cbe) + j
                        : reinterpret_cast<uint4*>(scales + (size_t)slot * L.nse * 2) + (j - cb);
    uint4* st = reinterpret_cast<uint4*>(staging + (size_t)m * staging_stride) + j;
    if (kGather)
      *st = *dev;
    else
      *dev = *st;
  }
}

}  // namespace moe

using namespace moe;

extern "C" size_t moe_adapt_workspace_bytes(const moe_layer* layer, int32_t max_swaps) {
  if (!layer || max_swaps < 0 || layer->n_experts < 1 || layer->n_experts > 1024) return 0;
  if (moe_workspace_bytes(layer, 1) == 0) return 0;   // the layer checks
  LayerDev L{};
  L.d = layer->d_model;
  L.F = layer->ffn;
  L.E = layer->n_experts;
  L.cbe = 3LL * L.F * L.d / kGroup * group_bytes(layer->bits);
  L.nse = 3LL * L.F * L.d / kGroup;
  return adapt_ws(L, max_swaps).total;
}

extern "C" moe_status moe_adapt_layout(const moe_layer* layer, float decay, int32_t max_swaps,
                                       int32_t* swaps_done_or_null, void* ws, size_t ws_bytes,
                                       void* stream) {
  if (!layer || !layer->route_counts || !ws || max_swaps < 0) return MOE_ERR_INVALID_ARG;
  if (!(decay >= 0.f && decay <= 1.f)) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_adapt_workspace_bytes(layer, max_swaps);
  if (need == 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MOE_ERR_MISALIGNED;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (!layer->codes || !layer->scales || !layer->expert_slot) return MOE_ERR_INVALID_ARG;
  moe_status s = check_device();
  if (s != MOE_OK) return s;
  LayerDev L{};
  L.d = layer->d_model;
  L.E = layer->n_experts;
  L.F = layer->ffn;
  L.k = layer->top_k;
  L.bits = layer->bits;
  L.Fs = layer->shared_ffn;
  L.codes = layer->codes;
  L.scales = layer->scales;
  L.cbe = 3LL * L.F * L.d / kGroup * group_bytes(L.bits);
  L.nse = 3LL * L.F * L.d / kGroup;
  const AdaptWs w = adapt_ws(L, max_swaps);
  char* base = static_cast<char*>(ws);
  Control* ctl = reinterpret_cast<Control*>(base);
  int32_t* n_moves = reinterpret_cast<int32_t*>(base + w.n_moves);
  int32_t* moves = reinterpret_cast<int32_t*>(base + w.moves);
  unsigned char* staging = reinterpret_cast<unsigned char*>(base + w.staging);
  const size_t stride = (((size_t)L.cbe + (size_t)L.nse * 2) + 255) & ~size_t(255);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  adapt_plan_kernel<<<1, kPlanThreads, 0, st>>>(L, const_cast<int32_t*>(layer->expert_slot),
                                                layer->route_counts, decay, max_swaps, n_moves,
                                                moves, swaps_done_or_null, ctl);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (max_swaps > 0) {
    const int grid = 2 * sm_count();
    adapt_copy_kernel<true><<<grid, 256, 0, st>>>(L, n_moves, moves, staging, stride);
    adapt_copy_kernel<false><<<grid, 256, 0, st>>>(L, n_moves, moves, staging, stride);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
