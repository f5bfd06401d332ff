/*
 * moe.h -- C ABI of the routed sparse-MoE block on B200 (sm_100a).
 *
 * What the block computes.  The Strata pages describe one layer of
 * Qwen3.8-Flash-Next as: a router scores the token against 512 experts and
 * picks 10, an always-on shared expert runs beside them, and the GPU adds the
 * results up before the next layer starts ("Strata open-source runtime: a 12GB
 * card runs the 125B Qwen3 model", section "the model itself"; "Why Strata is
 * fast on low-VRAM GPUs", sections "the problem" and "one token, three
 * workers").  Decode checks a verify window of up to 4 tokens in one pass
 * (same page, "guess first, then check"); prefill reads prompts in chunks of up
 * to 8192 tokens ("reading long prompts").  Experts are stored as low-bit
 * group-quantised weights ("the cost": Q2_0 / IQ3 expert files).
 *
 * Per token x (bf16, d values):
 *   logits[e] = sum_i x[i] * Wr[e][i] + b[e]                       (fp32)
 *   ids       = the top_k largest logits (plus router_pref, when given),
 *               largest first, equal values -> lower expert index, NaN below
 *               every number
 *   w[j]      = exp(logits[ids[j]] - logits[ids[0]]) / sum over the selected
 *   FFN_e(x)  = Wd_e (silu(Wg_e x) * (Wu_e x)),  silu(z) = z / (1 + e^-z)
 *   y         = FFN_shared(x) + sum_j w[j] * FFN_{ids[j]}(x)   -> bf16
 * with MOE_F_PRENORM the FFNs and the router see bf16(RMSNorm(x)) (eps 1e-6, no
 * weight) instead of x, and with MOE_F_RESIDUAL the output is x + y.
 *
 * Packed expert weights.  Each expert is Wg (ffn x d), Wu (ffn x d), Wd
 * (d x ffn), each R x K with K contracted, quantised in groups of 32
 * consecutive K elements: weight = fp16 scale * (code - 2^(bits-1)).
 *  - rows in tiles of 16; inside a tile, group words ordered group-major:
 *    word (c, r) at byte (c*16 + r) * 8 of the tile;
 *  - code j = 8m + 2t + h of a group: low two bits at bit 32h + 8t + 2m of
 *    the group's 8-byte little-endian word;
 *  - bits = 3: the high bit of code j at bit 16h + 4t + m of a 4-byte word;
 *    a tile holds all its 8-byte words (K/32*16*8 bytes), then all its 4-byte
 *    words in the same (c, r) order;
 *  - scales: fp16, one per (row, group), element c*16 + r of the tile's
 *    16*K/32 scales;
 *  - an expert = Wg tiles, Wu tiles, Wd tiles (codes), and the same order for
 *    its scales; expert e lives in slot expert_slot[e].
 *  Bytes per expert: codes 3*ffn*d/32 * (8 | 12), scales 3*ffn*d/32 * 2.
 *
 * Conventions for every call below.
 *  - Pointers marked "dev" are device memory owned by the caller; the library
 *    never allocates, frees or synchronises.  It enqueues kernels on `stream`
 *    (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *  - Row-major layouts, token dimension outermost.
 *  - Validation (null pointers, shapes, alignment, workspace size) happens on
 *    the host before any launch; a failed check returns its status and
 *    enqueues nothing.  MOE_OK means "enqueued": asynchronous faults surface
 *    at the caller's next synchronisation, and the kernels' own checks (bounded
 *    waits; range checks under MOE_F_DEBUG) set an error word in the
 *    workspace, read back with moe_workspace_error().
 *  - The workspace is caller-owned device memory of at least
 *    moe_workspace_bytes() bytes, 256-byte aligned, zeroed once with
 *    moe_workspace_init() before first use.  Kernels leave it ready for the
 *    next call.  Calls sharing one workspace must be ordered (same stream or
 *    explicit events).
 *  - Thread-safe for calls on distinct workspaces; stateless otherwise.
 *  - Limits: d_model % 32 == 0 and 32 <= d_model <= 4096; ffn, shared_ffn %
 *    32 == 0 and <= 4096; 1 <= top_k <= 16; top_k <= n_experts <= 1024;
 *    bits in {2, 3}; group == 32.
 *  - Alignment: x, y, codes, scales, shared_codes, shared_scales, router_w:
 *    16 bytes.
 *  - Precision: the expert products take fp16 operands.  Token values (after
 *    the optional RMSNorm) above 65,504 in magnitude saturate, and the kernels
 *    report them in the error word (kErrNonFinite, always checked); values
 *    below 6.1e-5 in magnitude keep only fp16-subnormal precision.  Routing
 *    logits are fp32; the output is accumulated in fp32 and rounded once to
 *    bf16.
 */
#ifndef MOE_H
#define MOE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad flag */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* a limit above is not met */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3,
  MOE_ERR_MISALIGNED = 4,
  MOE_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_CHECK = 6,       /* a kernel range check tripped (MOE_F_DEBUG) */
  MOE_ERR_TIMEOUT = 7,            /* a kernel's bounded wait ran out */
  MOE_ERR_NO_DEVICE = 8           /* no sm_100 device current */
} moe_status;

/* flags */
#define MOE_F_PRENORM 1u        /* router and experts see bf16(RMSNorm(x)) */
#define MOE_F_RESIDUAL 2u       /* y = x + MoE(.) */
#define MOE_F_DETERMINISTIC 4u  /* accepted; every path already combines in a fixed order */
#define MOE_F_DEBUG 8u          /* kernels range-check ids, slots and values */

/* One layer.  A host struct, read only during the call. */
typedef struct moe_layer_s {
  int32_t d_model;       /* d */
  int32_t n_experts;     /* E */
  int32_t ffn;           /* F, routed experts' hidden size */
  int32_t top_k;         /* k */
  int32_t bits;          /* 2 or 3 */
  int32_t group;         /* must be 32 */
  int32_t shared_ffn;    /* Fs; 0 = no shared expert */
  const float* router_w;        /* dev fp32 [E][d] */
  const float* router_bias;     /* dev fp32 [E] or NULL */
  const int32_t* expert_slot;   /* dev int32 [E]: expert -> slot, a permutation of 0..E-1 */
  const uint8_t* codes;         /* dev [E slots][3*F*d/32*(8|12)] */
  const uint16_t* scales;       /* dev fp16 bits [E slots][3*F*d/32] */
  const uint8_t* shared_codes;  /* dev [3*Fs*d/32*(8|12)] or NULL when Fs == 0 */
  const uint16_t* shared_scales;/* dev fp16 bits [3*Fs*d/32] or NULL when Fs == 0 */
  /* dev fp32 [E] or NULL: a per-expert selection bonus.  The selection ranks
   * logits[e] + router_pref[e] (fp32 add; same tie and NaN rules), while the
   * weights stay the softmax of the selected experts' logits.  This is the
   * pages' "the router prefers experts already on the card" (release 0.2.7 in
   * "Strata: a 12GB card runs 125B -- how the three storage tiers are
   * squeezed out", section 4, "how to choose against Ollama / LM Studio /
   * llama.cpp"): a positive bonus on a preferred set of experts.  NULL =
   * plain top-k. */
  const float* router_pref;
  /* dev fp32 [E] or NULL: routing counters for the adaptive slot layout.
   * When given, every selection made by the router (moe_route_topk and the
   * block forward) adds 1.0 to route_counts[expert] (atomic adds of ones:
   * exact below 2^24); moe_adapt_layout reads and decays them.  Selections
   * passed in by the caller (the expert-step calls) are not counted. */
  float* route_counts;
  /* host pointer or NULL: the layer the caller runs after this one.  Its
   * input-independent weights (router_w, shared_codes, shared_scales) are
   * prefetched into L2 (cp.async.bulk.prefetch.L2, spread over the thread
   * blocks) by this layer's decode expert step, so that the next layer's
   * router and shared expert read them from L2 instead of HBM.  A hint: the
   * results do not depend on it.  Read during the call like this struct; its
   * shape fields must pass the limits above and its pointers be 16-byte
   * aligned, else the call returns MOE_ERR_INVALID_ARG.  The pages overlap
   * the next layer's weight transfer with the current layer's compute in the
   * same way ("Strata illustrated", section on long prompts: the next
   * layer's experts stream in while the current layer computes). */
  const struct moe_layer_s* l2_next;
  /* dev bf16 bits [2][E][d] or NULL: the router weights split once into
   * hi = bf16(router_w) followed by lo = bf16(router_w - hi), as written by
   * moe_router_split().  When given, the tensor-core router of windows above
   * 8 tokens reads it instead of splitting router_w into the workspace on
   * every call (same logits, bit for bit).  The caller keeps it in step with
   * router_w.  16-byte aligned, else MOE_ERR_MISALIGNED. */
  const uint16_t* router_w_split;
} moe_layer;

/* Split the layer's fp32 router weights into the bf16 hi and lo parts the
 * tensor-core router multiplies (out: dev bf16 bits [2][E][d], 16-byte
 * aligned, caller-owned; enqueued on stream).  Meant for once per layer at
 * load time: set the result as moe_layer.router_w_split.  The router's
 * accuracy argument is in the comment of the router for long windows: the
 * residual of the two terms is below 2^-16 |Wr|. */
moe_status moe_router_split(const moe_layer* layer, uint16_t* out, void* stream);

/* Bytes of workspace the calls below need for up to max_tokens tokens
 * (0 on invalid arguments).  The decode path (moe_route_topk with T <= 8,
 * moe_expert_ffn_decode, moe_block_forward with T <= 8 on a layer the decode
 * kernels take) uses only a leading part of the layout and accepts any
 * workspace at least that large; the prefill path needs the full size. */
size_t moe_workspace_bytes(const moe_layer* layer, int32_t max_tokens);

/* Zero a workspace (enqueued on stream).  Needed once after allocation. */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Copy the workspace's device error word to *code_out (0 = none) and clear it.
 * Synchronises `stream` (a debugging aid, not for the hot path).  Returns
 * MOE_ERR_TIMEOUT / MOE_ERR_DEVICE_CHECK when the word was set. */
moe_status moe_workspace_error(void* ws, size_t ws_bytes, uint32_t* code_out, void* stream);

/* Set the limit of the kernels' bounded waits for calls on this workspace
 * (enqueued on stream; a one-thread kernel, so it may be graph-captured).
 * Every wait of a kernel on a pipeline barrier (a shared-memory stage, a
 * tensor-memory accumulator, an asynchronous copy) gives up after limit_us
 * microseconds of the GPU's global timer, records MOE_ERR_TIMEOUT in the
 * error word and stops issuing work; before its thread block ends it waits
 * for the copies and tensor-core operations it already issued.  The outputs of
 * a call that timed out are undefined; the workspace stays usable.
 * limit_us = 0 restores the default of one second; other values from 1,000
 * (1 ms: a wait reads the limit only once it has lasted that long) to
 * 60,000,000 (60 s), else MOE_ERR_INVALID_ARG.  moe_workspace_init() restores the default.  The
 * pages' engine has no counterpart: this bounds a stuck pipeline. */
moe_status moe_workspace_set_wait_limit(void* ws, size_t ws_bytes, uint32_t limit_us, void* stream);

/* Test switch for the bounded-wait path (enqueued on stream like the call
 * above).  site = 1: in calls that pass MOE_F_DEBUG and run the prefill
 * expert step (moe_expert_ffn_prefill, or moe_block_forward with T > 32), one
 * epilogue thread of thread block 0 of the gate/up GEMM skips its plain
 * arrive on the barrier that frees the first tensor-memory accumulator, so
 * the MMA issuer's wait before that block's third work item runs out (a call
 * with at least 3 x 148 gate/up work items, e.g. 64 tokens of a 512-expert
 * layer, reaches it) and the call ends with MOE_ERR_TIMEOUT in the error word
 * after a few wait limits; the copies and MMAs already issued complete
 * before the thread block ends.  Calls without MOE_F_DEBUG ignore the
 * switch.  site = 0 turns it off; other values return
 * MOE_ERR_INVALID_ARG.  moe_workspace_init() turns it off.  No counterpart
 * in the pages: it exists to test the error path without a fault. */
moe_status moe_workspace_set_debug_withhold(void* ws, size_t ws_bytes, uint32_t site,
                                            void* stream);

/* Router + top-k + softmax renormalisation for T tokens.
 *  x_bf16: dev bf16 [T][d].  flags: MOE_F_PRENORM and MOE_F_DEBUG honoured.
 *  logits_or_null: dev fp32 [T][E], written when non-NULL.
 *  topk_ids: dev int32 [T][k] (largest first); topk_w: dev fp32 [T][k].
 *  T = 0 enqueues nothing. */
moe_status moe_route_topk(const moe_layer* layer, const void* x_bf16, int32_t T, uint32_t flags,
                          float* logits_or_null, int32_t* topk_ids, float* topk_w, void* ws,
                          size_t ws_bytes, void* stream);

/* Decode / verify-window expert step for 1 <= T <= 8 tokens: the selected
 * experts (deduplicated across the window) and the shared expert, combined
 * with the routing weights.  Weight bytes are streamed once per call.
 *  topk_ids/topk_w: dev, as written by moe_route_topk.  y_bf16: dev bf16 [T][d]
 *  (may not alias x).  flags: PRENORM, RESIDUAL, DEBUG.
 *  Returns MOE_ERR_UNSUPPORTED_SHAPE, before enqueuing anything, for T > 8 and
 *  for experts too wide for the kernels' shared-memory stages: each of 16
 *  warps stages one expert's whole down-projection tile with its hidden
 *  vectors, so the limit on max(ffn, shared_ffn) falls as T grows (d 2048 and
 *  512 experts: up to 1888 (2-bit) / 1472 (3-bit) at T = 1, 608 / 576 at
 *  T = 8). */
moe_status moe_expert_ffn_decode(const moe_layer* layer, const void* x_bf16, int32_t T,
                                 const int32_t* topk_ids, const float* topk_w, void* y_bf16,
                                 uint32_t flags, void* ws, size_t ws_bytes, void* stream);

/* Prefill expert step for T >= 1 tokens: tokens bucketed per expert (ascending
 * token order inside each expert), tensor-core grouped GEMMs with the
 * dequantisation fused into the operand tiles, shared expert over all tokens,
 * routing-weighted combine.
 *  bucket_offsets_or_null: dev int32 [E+1], written when non-NULL (exclusive
 *  scan of per-expert counts).  bucket_entries_or_null: dev int32 [T*k],
 *  written when non-NULL: for each expert its entries t*k + j, tokens
 *  ascending.  flags: PRENORM, RESIDUAL, DETERMINISTIC, DEBUG. */
moe_status moe_expert_ffn_prefill(const moe_layer* layer, const void* x_bf16, int32_t T,
                                  const int32_t* topk_ids, const float* topk_w, void* y_bf16,
                                  int32_t* bucket_offsets_or_null, int32_t* bucket_entries_or_null,
                                  uint32_t flags, void* ws, size_t ws_bytes, void* stream);

/* The whole block: moe_route_topk, then the decode step for T <= 8 when the
 * layer fits the decode kernels (faster than the prefill step at every window
 * it supports) and the prefill step otherwise.  Windows of 9..32 tokens run
 * as consecutive decode windows of up to 8 tokens (router and decode step per
 * window), which measured faster than the prefill step there (decode layer,
 * 2-bit: 63 vs 130 us at T = 9, 171 vs 182 us at T = 32; the prefill step
 * wins from T = 40).  Routing lists live in the workspace; for 9..32 tokens
 * the decode part of the workspace suffices. */
moe_status moe_block_forward(const moe_layer* layer, const void* x_bf16, int32_t T, void* y_bf16,
                             uint32_t flags, void* ws, size_t ws_bytes, void* stream);

/* moe_block_forward for a decode window (0 <= T <= 4) without a caller
 * workspace: the scratch is a 2 MiB array in the library's device memory, one
 * per device.  The Strata pages have no counterpart; this is for callers that
 * cannot allocate or own a workspace (a plain C host without a device
 * allocator, a step loop that must not call cudaMalloc, which synchronises the
 * device).
 *  - Allocates nothing.  The first call on a device (with that device
 *    current) looks up the array's address with cudaGetSymbolAddress; make
 *    that first call before any stream capture.  The address is cached with
 *    the id of the CUDA context it came from and looked up again when the
 *    current context changes (after a device reset, for instance).
 *  - Every call that passes validation first zeroes the array's 256-byte
 *    control block with an enqueued cudaMemsetAsync (error word, counters);
 *    nothing else has to be initialised.  Device-side error bits cannot be
 *    read back through this entry point; use moe_block_forward with a
 *    workspace to inspect them.
 *  - One scratch per device: calls on the same device must be ordered (one
 *    stream, or events); calls that overlap on the GPU race on the scratch.
 *  - Shapes whose workspace (moe_workspace_bytes(layer, T)) exceeds 2 MiB
 *    return MOE_ERR_WORKSPACE_TOO_SMALL; T > 4 returns
 *    MOE_ERR_UNSUPPORTED_SHAPE; both before anything is enqueued.  A layer
 *    too wide for the decode kernels (see moe_expert_ffn_decode) takes the
 *    prefill step, whose full workspace must then fit in the 2 MiB.
 *  - Status codes match moe_block_forward's (MOE_ERR_NO_DEVICE without a
 *    current sm_100 device). */
moe_status moe_block_forward_noalloc(const moe_layer* layer, const void* x_bf16, int32_t T,
                                     void* y_bf16, uint32_t flags, void* stream);

/* Adaptive frequency-ordered slot layout.  The pages' expert cache keeps
 * counting the routing with exponential decay and swaps new hot experts in, at
 * most 96 swaps per 4 rounds ("Strata: Run a 125B Model on a 12 GB GPU with
 * MoE Expert Hot Cache", section "How It Works"; "Strata illustrated",
 * section on the expert cache).  With every expert in HBM the "cache" is the
 * slot order: this call ranks the experts by layer->route_counts (descending,
 * equal counts by lower expert index), walks the ranks and swaps the expert
 * of rank r into slot r until max_swaps swaps are made, moves the packed
 * bytes (codes and scales) of the affected slots, rewrites expert_slot, and
 * multiplies every count by decay (0 <= decay <= 1).  Results of the block do
 * not depend on the slot order, so outputs stay bit-identical.
 *  - Rewrites layer->codes, ->scales and ->expert_slot in place (they must be
 *    writable device memory) and layer->route_counts (required).
 *  - ws: at least moe_adapt_workspace_bytes(layer, max_swaps) bytes,
 *    256-byte aligned (staging for 2*max_swaps slots).
 *  - swaps_done_or_null: dev int32, receives the number of swaps made.
 *  - Enqueued on stream after the work before it, without programmatic
 *    overlap; a slot table that is not a permutation moves nothing and sets
 *    the range bit in the workspace's error word (moe_workspace_error). */
size_t moe_adapt_workspace_bytes(const moe_layer* layer, int32_t max_swaps);
moe_status moe_adapt_layout(const moe_layer* layer, float decay, int32_t max_swaps,
                            int32_t* swaps_done_or_null, void* ws, size_t ws_bytes, void* stream);

const char* moe_status_string(moe_status status);

/* Library build information (a static string). */
const char* moe_build_info(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
