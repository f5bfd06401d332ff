// noalloc.cu -- a decode-window block forward whose scratch is a file-scope
// device array instead of a caller-supplied workspace.
//
// The Strata pages have no counterpart to this call: it exists for callers
// that cannot allocate or own a device workspace.  Examples are a C host that
// links only this library and has no device allocator at hand, and a serving
// loop that must not call cudaMalloc (which synchronises the device) between
// steps.  Every other entry point takes a caller-owned workspace.
//
// The scratch is one static array per device (kNoAllocScratchBytes, 2 MiB):
// enough for the control block, logits, routing lists and decode partial sums
// of a T <= 4 window at the shapes of the Strata layer (d = 2048, 512 experts,
// ffn 512, top-10).  Larger needs are rejected with
// MOE_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"

namespace moe {

constexpr size_t kNoAllocScratchBytes = 2u << 20;
constexpr int kNoAllocMaxDevices = 64;

// Zero at module load.  Each call also zeroes the control block at its start
// (an enqueued memset, no allocation), so an error bit set by an earlier call
// does not persist and the self-resetting counters start from zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// The device address of the array, per device, together with the unique id of
// the CUDA context it was looked up in.  A device reset (or any teardown of the
// primary context) loads the module again, possibly at another address; a
// changed context id triggers a new lookup.
struct ScratchAddr {
  unsigned long long ctx_id = 0;
  void* ptr = nullptr;
};
ScratchAddr g_addr[kNoAllocMaxDevices];
std::mutex g_addr_mu;

PFN_cuCtxGetCurrent_v4000 g_get_ctx = nullptr;
PFN_cuCtxGetId_v12000 g_get_id = nullptr;

bool load_ctx_entry_points() {
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    cudaGetLastError();
  });
  return g_get_ctx && g_get_id;
}

// Address of this device's copy of the scratch array in the current context,
// or nullptr on failure.  Called with `dev` current.
void* scratch_address(int dev) {
  if (!load_ctx_entry_points()) return nullptr;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_get_ctx(&ctx) != CUDA_SUCCESS || !ctx || g_get_id(ctx, &id) != CUDA_SUCCESS) return nullptr;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  ScratchAddr& a = g_addr[dev];
  if (a.ptr && a.ctx_id == id) return a.ptr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return nullptr;
  }
  a.ptr = p;
  a.ctx_id = id;
  return p;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_block_forward_noalloc(const moe_layer* layer, const void* x_bf16,
                                                int32_t T, void* y_bf16, uint32_t flags,
                                                void* stream) {
  using namespace moe;
  if (T < 0 || T > 4) return MOE_ERR_UNSUPPORTED_SHAPE;
  // the same device check as every other entry point, before any lookup
  moe_status s = check_device();
  if (s != MOE_OK) return s;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  void* ws = scratch_address(dev);
  if (!ws) return MOE_ERR_CUDA;
  // every argument is validated before anything is enqueued; a call that
  // passes zeroes the scratch's control block first (error word, counters)
  return block_forward(layer, x_bf16, T, y_bf16, flags, ws, kNoAllocScratchBytes, stream, true);
}
