// moe_api.cu -- the C ABI declared in include/moe.h: argument validation,
// workspace layout and the kernel launch sequence of each entry point.
#include <cuda_runtime.h>
#include <stdio.h>

#include "internal.h"

#define MOE_STR_(x) #x
#define MOE_STR(x) MOE_STR_(x)

namespace moe {

cudaError_t launch_prep_tokens(const uint16_t* x, int T, int d, uint32_t flags, uint16_t* xn,
                               __half* x16, Control* ctl, cudaStream_t st);
size_t decode_hw_bytes(const LayerDev& L, int T);
size_t prefill_ws_bytes(const LayerDev& L, int T, size_t* parts);

namespace {
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
int g_dev_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 not an sm_100 device

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

moe_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  if (g_dev_ok[dev] == 0) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_NO_DEVICE;
    }
    g_sm_count[dev] = sms;
    g_dev_ok[dev] = (major == 10) ? 1 : -1;
  }
  return g_dev_ok[dev] == 1 ? MOE_OK : MOE_ERR_NO_DEVICE;
}

namespace {

moe_status validate_own(const moe_layer* l) {
  if (!l) return MOE_ERR_INVALID_ARG;
  if (l->group != kGroup) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (l->bits != 2 && l->bits != 3) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (l->d_model < 32 || l->d_model > 4096 || l->d_model % 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (l->ffn < 32 || l->ffn > 4096 || l->ffn % 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (l->shared_ffn < 0 || l->shared_ffn > 4096 || l->shared_ffn % 32)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (l->top_k < 1 || l->top_k > 16 || l->n_experts < l->top_k || l->n_experts > 1024)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!l->router_w || !l->expert_slot || !l->codes || !l->scales) return MOE_ERR_INVALID_ARG;
  if (l->shared_ffn > 0 && (!l->shared_codes || !l->shared_scales)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(l->router_w) || !aligned16(l->codes) || !aligned16(l->scales))
    return MOE_ERR_MISALIGNED;
  if (l->shared_ffn > 0 && (!aligned16(l->shared_codes) || !aligned16(l->shared_scales)))
    return MOE_ERR_MISALIGNED;
  if (l->router_w_split && !aligned16(l->router_w_split)) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

// The layer, and the next layer named for the L2 prefetch (its own fields only).
moe_status validate_layer(const moe_layer* l) {
  const moe_status s = validate_own(l);
  if (s != MOE_OK) return s;
  if (l->l2_next && validate_own(l->l2_next) != MOE_OK) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

LayerDev to_dev(const moe_layer* l) {
  LayerDev L;
  L.d = l->d_model;
  L.E = l->n_experts;
  L.F = l->ffn;
  L.k = l->top_k;
  L.bits = l->bits;
  L.Fs = l->shared_ffn;
  L.Wr = l->router_w;
  L.bias = l->router_bias;
  L.slot = l->expert_slot;
  L.codes = l->codes;
  L.scales = l->scales;
  L.scodes = l->shared_codes;
  L.sscales = l->shared_scales;
  L.pref = l->router_pref;
  L.counts = l->route_counts;
  L.wsplit = l->router_w_split;
  L.cbe = 3LL * L.F * L.d / kGroup * group_bytes(L.bits);
  L.nse = 3LL * L.F * L.d / kGroup;
  for (int r = 0; r < 3; ++r) {
    L.pf[r] = nullptr;
    L.pfb[r] = 0;
  }
  if (const moe_layer* n = l->l2_next) {   // checked by validate_layer
    const long long sg = 3LL * n->shared_ffn * n->d_model / kGroup;
    L.pf[0] = reinterpret_cast<const char*>(n->router_w);
    L.pfb[0] = (unsigned)((long long)n->n_experts * n->d_model * 4);
    L.pf[1] = reinterpret_cast<const char*>(n->shared_codes);
    L.pfb[1] = n->shared_codes ? (unsigned)(sg * group_bytes(n->bits)) : 0u;
    L.pf[2] = reinterpret_cast<const char*>(n->shared_scales);
    L.pfb[2] = n->shared_scales ? (unsigned)(sg * 2) : 0u;
  }
  return L;
}

moe_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  cudaGetLastError();
  return MOE_ERR_CUDA;
}

__global__ void set_word_kernel(uint32_t* p, uint32_t v) { *p = v; }

// One word of a workspace control block, written in stream order.
moe_status set_control_word(uint32_t* p, uint32_t v, cudaStream_t st) {
  set_word_kernel<<<1, 1, 0, st>>>(p, v);
  return from_cuda(cudaGetLastError());
}

// Common preamble of every compute entry point.
moe_status preamble(const moe_layer* layer, int32_t T, const void* x, void* ws, size_t ws_bytes,
                    bool decode_path,
                    LayerDev* L, WsLayout* lay) {
  moe_status s = validate_layer(layer);
  if (s != MOE_OK) return s;
  if (T < 0 || !ws || !x) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_MISALIGNED;
  *L = to_dev(layer);
  *lay = ws_layout(*L, T);
  if (ws_bytes < (decode_path ? lay->decode_total : lay->total)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}
}  // namespace

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < kMaxDevices && g_sm_count[dev] > 0) ? g_sm_count[dev] : 148;
}

WsLayout ws_layout(const LayerDev& L, int T) {
  WsLayout w = {};
  size_t o = 0;
  const size_t Tn = T > 0 ? (size_t)T : 1;
  w.ctl = o;
  o += align256(sizeof(Control));
  w.logits = o;
  o += align256(Tn * L.E * sizeof(float));
  w.ids = o;
  o += align256(Tn * L.k * sizeof(int32_t));
  w.w = o;
  o += align256(Tn * L.k * sizeof(float));
  w.hw = o;
  o += align256(decode_hw_bytes(L, T < kMaxDecodeT ? (int)Tn : kMaxDecodeT));
  w.decode_total = o;   // the decode path (router for T <= 8, decode step) uses no more
  if (T > 0) {
    size_t parts[16];
    prefill_ws_bytes(L, T, parts);
    w.xn = o;
    o += align256(parts[0]);
    w.x16 = o;
    o += align256(parts[1]);
    w.counts = o;
    o += align256(parts[2]);
    w.offsets = o;
    o += align256(parts[3]);
    w.entries = o;
    o += align256(parts[4]);
    w.blockcnt = o;
    o += align256(parts[5]);
    w.tiles = o;
    o += align256(parts[6]);
    w.h = o;
    o += align256(parts[7]);
    w.yacc = o;
    o += align256(parts[8]);
    w.xperm = o;
    o += align256(parts[9]);
  }
  if (T > kMaxDecodeT) {
    w.wsplit = o;
    o += align256((size_t)2 * L.E * L.d * sizeof(uint16_t));
  }
  w.total = o;
  return w;
}


// The block forward behind moe_block_forward (and the allocation-free entry
// point): every argument is validated first; with clear_control the
// workspace's control block is zeroed on the stream just before the kernels.
moe_status block_forward(const moe_layer* layer, const void* x_bf16, int32_t T, void* y_bf16,
                         uint32_t flags, void* ws, size_t ws_bytes, void* stream,
                         bool clear_control) {
  LayerDev L;
  WsLayout lay;
  if (!y_bf16 || !layer) return MOE_ERR_INVALID_ARG;
  // the decode kernels are faster up to their 8-token limit, for layers whose
  // experts fit their shared-memory stages; windows of 9..kSubWindowMaxT
  // tokens run as consecutive decode windows of up to 8 tokens, which was
  // measured faster than the prefill pipeline there (decode layer, 2-bit:
  // 63 vs 130 us at T = 9, 86 vs 151 us at T = 16, 171 vs 182 us at T = 32,
  // 214 vs 193 us at T = 40)
  const int Fmax = layer->ffn > layer->shared_ffn ? layer->ffn : layer->shared_ffn;
  const bool dec = T <= kMaxDecodeT &&
                   (T == 0 || decode_fits(layer->d_model, layer->n_experts, Fmax, layer->bits, T));
  const bool sub = T > kMaxDecodeT && T <= kSubWindowMaxT &&
                   decode_fits(layer->d_model, layer->n_experts, Fmax, layer->bits, kMaxDecodeT);
  moe_status s = preamble(layer, T, x_bf16, ws, ws_bytes, dec || sub, &L, &lay);
  if (s != MOE_OK) return s;
  if (y_bf16 == x_bf16) return MOE_ERR_INVALID_ARG;
  if (flags & ~(MOE_F_PRENORM | MOE_F_RESIDUAL | MOE_F_DETERMINISTIC | MOE_F_DEBUG))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_bf16)) return MOE_ERR_MISALIGNED;
  if ((s = check_device()) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  char* w = static_cast<char*>(ws);
  if (clear_control) {
    s = from_cuda(cudaMemsetAsync(w + lay.ctl, 0, sizeof(Control), static_cast<cudaStream_t>(stream)));
    if (s != MOE_OK) return s;
  }
  int32_t* ids = reinterpret_cast<int32_t*>(w + lay.ids);
  float* wt = reinterpret_cast<float*>(w + lay.w);
  if (sub) {
    // consecutive decode windows of up to 8 tokens, stream-ordered on the
    // workspace's decode regions
    const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
    uint16_t* y = static_cast<uint16_t*>(y_bf16);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Control* ctl = reinterpret_cast<Control*>(w + lay.ctl);
    for (int t0 = 0; t0 < T; t0 += kMaxDecodeT) {
      const int n = T - t0 < kMaxDecodeT ? T - t0 : kMaxDecodeT;
      const WsLayout ln = ws_layout(L, n);
      int32_t* ids_n = reinterpret_cast<int32_t*>(w + ln.ids);
      float* w_n = reinterpret_cast<float*>(w + ln.w);
      cudaError_t e = launch_router_small(L, x + (size_t)t0 * L.d, n, flags,
                                          reinterpret_cast<float*>(w + ln.logits), ids_n, w_n,
                                          ctl, st);
      if (e == cudaSuccess)
        e = launch_decode(L, x + (size_t)t0 * L.d, n, ids_n, w_n, y + (size_t)t0 * L.d, flags,
                          w, ln, st);
      if (e != cudaSuccess) return from_cuda(e);
    }
    return MOE_OK;
  }
  s = moe_route_topk(layer, x_bf16, T, flags, nullptr, ids, wt, ws, ws_bytes, stream);
  if (s != MOE_OK) return s;
  if (dec)
    return moe_expert_ffn_decode(layer, x_bf16, T, ids, wt, y_bf16, flags, ws, ws_bytes, stream);
  return moe_expert_ffn_prefill(layer, x_bf16, T, ids, wt, y_bf16, nullptr, nullptr, flags, ws,
                                ws_bytes, stream);
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_bytes(const moe_layer* layer, int32_t max_tokens) {
  if (validate_layer(layer) != MOE_OK || max_tokens < 0) return 0;
  return ws_layout(to_dev(layer), max_tokens).total;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < sizeof(Control)) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MOE_ERR_MISALIGNED;
  return from_cuda(cudaMemsetAsync(ws, 0, sizeof(Control), static_cast<cudaStream_t>(stream)));
}

moe_status moe_workspace_error(void* ws, size_t ws_bytes, uint32_t* code_out, void* stream) {
  if (!ws || ws_bytes < sizeof(Control)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t code = 0;
  Control* ctl = static_cast<Control*>(ws);
  cudaError_t e = cudaMemcpyAsync(&code, &ctl->err, sizeof(code), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && code) e = cudaMemsetAsync(&ctl->err, 0, sizeof(uint32_t), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return from_cuda(e);
  if (code_out) *code_out = code;
  if (code & kErrTimeout) return MOE_ERR_TIMEOUT;
  if (code) return MOE_ERR_DEVICE_CHECK;
  return MOE_OK;
}

moe_status moe_router_split(const moe_layer* layer, uint16_t* out, void* stream) {
  moe_status s = validate_layer(layer);
  if (s != MOE_OK) return s;
  if (!out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out)) return MOE_ERR_MISALIGNED;
  if ((s = check_device()) != MOE_OK) return s;
  const size_t n = (size_t)layer->n_experts * layer->d_model;
  return from_cuda(launch_split_router(layer->router_w, layer->n_experts, layer->d_model, out,
                                       out + n, static_cast<cudaStream_t>(stream)));
}

moe_status moe_workspace_set_wait_limit(void* ws, size_t ws_bytes, uint32_t limit_us,
                                        void* stream) {
  if (!ws || ws_bytes < sizeof(Control) || limit_us > 60000000u ||
      (limit_us != 0 && limit_us < kWaitFloorNs / 1000))
    return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MOE_ERR_MISALIGNED;
  moe_status s = check_device();
  if (s != MOE_OK) return s;
  return set_control_word(&static_cast<Control*>(ws)->wait_limit_us, limit_us,
                          static_cast<cudaStream_t>(stream));
}

moe_status moe_workspace_set_debug_withhold(void* ws, size_t ws_bytes, uint32_t site,
                                            void* stream) {
  if (!ws || ws_bytes < sizeof(Control) || site > kWithholdPrefillArrive)
    return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MOE_ERR_MISALIGNED;
  moe_status s = check_device();
  if (s != MOE_OK) return s;
  return set_control_word(&static_cast<Control*>(ws)->debug_withhold, site,
                          static_cast<cudaStream_t>(stream));
}

moe_status moe_route_topk(const moe_layer* layer, const void* x_bf16, int32_t T, uint32_t flags,
                          float* logits_or_null, int32_t* topk_ids, float* topk_w, void* ws,
                          size_t ws_bytes, void* stream) {
  LayerDev L;
  WsLayout lay;
  if (!topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if (flags & ~(MOE_F_PRENORM | MOE_F_RESIDUAL | MOE_F_DETERMINISTIC | MOE_F_DEBUG))
    return MOE_ERR_INVALID_ARG;
  moe_status s = preamble(layer, T, x_bf16, ws, ws_bytes, T <= kMaxDecodeT, &L, &lay);
  if (s != MOE_OK) return s;
  if ((s = check_device()) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  char* w = static_cast<char*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Control* ctl = reinterpret_cast<Control*>(w + lay.ctl);
  float* logits = logits_or_null ? logits_or_null : reinterpret_cast<float*>(w + lay.logits);
  const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
  if (T <= kMaxDecodeT)
    return from_cuda(launch_router_small(L, x, T, flags, logits, topk_ids, topk_w, ctl, st));
  // large T: prenorm into xn first, the router reads bf16
  const uint16_t* xr = x;
  if (flags & MOE_F_PRENORM) {
    cudaError_t e = launch_prep_tokens(x, T, L.d, flags, reinterpret_cast<uint16_t*>(w + lay.xn),
                                       reinterpret_cast<__half*>(w + lay.x16), ctl, st);
    if (e != cudaSuccess) return from_cuda(e);
    xr = reinterpret_cast<const uint16_t*>(w + lay.xn);
  }
  return from_cuda(launch_router_large(L, xr, T, flags, logits, topk_ids, topk_w,
                                       reinterpret_cast<uint16_t*>(w + lay.wsplit), ctl, st));
}

moe_status moe_expert_ffn_decode(const moe_layer* layer, const void* x_bf16, int32_t T,
                                 const int32_t* topk_ids, const float* topk_w, void* y_bf16,
                                 uint32_t flags, void* ws, size_t ws_bytes, void* stream) {
  LayerDev L;
  WsLayout lay;
  if (!topk_ids || !topk_w || !y_bf16) return MOE_ERR_INVALID_ARG;
  if (flags & ~(MOE_F_PRENORM | MOE_F_RESIDUAL | MOE_F_DETERMINISTIC | MOE_F_DEBUG))
    return MOE_ERR_INVALID_ARG;
  if (T > kMaxDecodeT) return MOE_ERR_UNSUPPORTED_SHAPE;
  moe_status s = preamble(layer, T, x_bf16, ws, ws_bytes, true, &L, &lay);
  if (s != MOE_OK) return s;
  if (T > 0 && !decode_fits(L.d, L.E, L.F > L.Fs ? L.F : L.Fs, L.bits, T))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(y_bf16)) return MOE_ERR_MISALIGNED;
  if (y_bf16 == x_bf16) return MOE_ERR_INVALID_ARG;
  if ((s = check_device()) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  return from_cuda(launch_decode(L, static_cast<const uint16_t*>(x_bf16), T, topk_ids, topk_w,
                                 static_cast<uint16_t*>(y_bf16), flags, static_cast<char*>(ws), lay,
                                 static_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn_prefill(const moe_layer* layer, const void* x_bf16, int32_t T,
                                  const int32_t* topk_ids, const float* topk_w, void* y_bf16,
                                  int32_t* bucket_offsets_or_null, int32_t* bucket_entries_or_null,
                                  uint32_t flags, void* ws, size_t ws_bytes, void* stream) {
  LayerDev L;
  WsLayout lay;
  if (!topk_ids || !topk_w || !y_bf16) return MOE_ERR_INVALID_ARG;
  if (flags & ~(MOE_F_PRENORM | MOE_F_RESIDUAL | MOE_F_DETERMINISTIC | MOE_F_DEBUG))
    return MOE_ERR_INVALID_ARG;
  moe_status s = preamble(layer, T, x_bf16, ws, ws_bytes, false, &L, &lay);
  if (s != MOE_OK) return s;
  if (!aligned16(y_bf16)) return MOE_ERR_MISALIGNED;
  if (y_bf16 == x_bf16) return MOE_ERR_INVALID_ARG;
  if ((s = check_device()) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  return from_cuda(launch_prefill(L, static_cast<const uint16_t*>(x_bf16), T, topk_ids, topk_w,
                                  static_cast<uint16_t*>(y_bf16), bucket_offsets_or_null,
                                  bucket_entries_or_null, flags, static_cast<char*>(ws), lay,
                                  static_cast<cudaStream_t>(stream)));
}

moe_status moe_block_forward(const moe_layer* layer, const void* x_bf16, int32_t T, void* y_bf16,
                             uint32_t flags, void* ws, size_t ws_bytes, void* stream) {
  return moe::block_forward(layer, x_bf16, T, y_bf16, flags, ws, ws_bytes, stream, false);
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_MISALIGNED: return "misaligned pointer";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_CHECK: return "device-side check failed";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_NO_DEVICE: return "no sm_100 device";
  }
  return "unknown status";
}

const char* moe_build_info(void) {
  return "routed-moe sm_100a; nvcc " MOE_STR(__CUDACC_VER_MAJOR__) "." MOE_STR(__CUDACC_VER_MINOR__);
}

}  // extern "C"
