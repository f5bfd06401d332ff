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
// enough for the control block, logits, routing lists and decode hidden
// fragments of a T <= 4 window at the shapes of the Strata layer (d = 2048,
// 512 experts, ffn 512, top-10 need about 0.6 MB).  Larger needs are rejected
// with MOE_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.
#include <atomic>

#include "internal.h"

namespace moe {

constexpr size_t kNoAllocScratchBytes = 2u << 20;
constexpr int kNoAllocMaxDevices = 64;

// Zero at module load, which is the state the workspace control block must
// start in (error word, self-resetting CTA counters); the kernels leave it that
// way after every call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static std::atomic<void*> g_noalloc_ptr[kNoAllocMaxDevices];

}  // namespace moe

extern "C" moe_status moe_block_forward_noalloc(const moe_layer* layer, const void* x_bf16,
                                                int32_t T, void* y_bf16, uint32_t flags,
                                                void* stream) {
  using namespace moe;
  if (T < 0 || T > 4) return MOE_ERR_UNSUPPORTED_SHAPE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  void* ws = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (!ws) {
    // once per device, with that device current: the address of this
    // device's copy of the array
    if (cudaGetSymbolAddress(&ws, g_noalloc_scratch) != cudaSuccess || !ws) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    g_noalloc_ptr[dev].store(ws, std::memory_order_release);
  }
  return moe_block_forward(layer, x_bf16, T, y_bf16, flags, ws, kNoAllocScratchBytes, stream);
}
