// internal.h -- host-side declarations shared by the library's translation units.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "moe.h"

namespace moe {

// A layer as the kernels receive it (by value).
struct LayerDev {
  int d, E, F, k, bits, Fs;
  const float* Wr;
  const float* bias;
  const int32_t* slot;
  const uint8_t* codes;
  const uint16_t* scales;
  const uint8_t* scodes;
  const uint16_t* sscales;
  const float* pref;   // selection bonus [E] or nullptr
  float* counts;       // routing counters [E] or nullptr
  const uint16_t* wsplit;   // router weights split into bf16 hi, lo [2][E][d] or nullptr
  const char* pf[3];   // L2 prefetch ranges (the next layer's router and shared expert)
  unsigned pfb[3];     // their bytes (multiples of 16; 0 = none)
  long long cbe;   // codes bytes per routed expert
  long long nse;   // scales per routed expert
};

__host__ __device__ inline int group_bytes(int bits) { return bits == 2 ? 8 : 12; }
// codes bytes of an R x K matrix
__host__ __device__ inline long long mat_codes_bytes(int R, int K, int bits) {
  return (long long)(R / kTileRows) * (K / kGroup) * kTileRows * group_bytes(bits);
}

// Workspace layout for T tokens (byte offsets; 256-aligned).
struct WsLayout {
  size_t ctl;        // Control
  size_t logits;     // fp32 [T][E]
  size_t ids;        // int32 [T][k]
  size_t w;          // fp32 [T][k]
  size_t hw;         // decode: fp16 fragments [(U_max+1)][Fmax/32][32][8]
  size_t xn;         // prefill: bf16 [T][d] (PRENORM)
  size_t x16;        // prefill: fp16 [T][d]
  size_t counts;     // prefill: int32 [E+1]
  size_t offsets;    // prefill: int32 [E+2]
  size_t entries;    // prefill: int32 [T*k]
  size_t blockcnt;   // prefill: int32 [nblk][E]
  size_t tiles;      // prefill: int32 work list
  size_t h;          // prefill: fp16 hidden [rows][Fmax]
  size_t yacc;       // (unused, zero bytes)
  size_t xperm;      // prefill: fp16 [T*(k+1)][d]: xperm (GEMM1 operand), then ybuf (GEMM2 output)
  size_t wsplit;     // T > decode window: router weights as bf16 hi and lo [2][E][d]
  size_t decode_total;   // bytes the decode path needs (a prefix of the layout)
  size_t total;
};
WsLayout ws_layout(const LayerDev& L, int T);

// launchers (return cudaError_t of the launch)
cudaError_t launch_router_small(const LayerDev& L, const uint16_t* x, int T, uint32_t flags,
                                float* logits, int32_t* ids, float* w, Control* ctl,
                                cudaStream_t st);
cudaError_t launch_router_large(const LayerDev& L, const uint16_t* x, int T, uint32_t flags,
                                float* logits, int32_t* ids, float* w, uint16_t* wsplit,
                                Control* ctl, cudaStream_t st);
cudaError_t launch_router_tc(const LayerDev& L, const uint16_t* x, int T, float* logits,
                             uint16_t* hi, uint16_t* lo, bool split, Control* ctl,
                             cudaStream_t st);
cudaError_t launch_split_router(const float* Wr, int E, int d, uint16_t* hi, uint16_t* lo,
                                cudaStream_t st);
bool decode_fits(int d, int E, int Fmax, int bits, int T);
// Widest window the block forward runs as consecutive decode windows of up
// to kMaxDecodeT tokens (the measured crossover to the prefill pipeline).
constexpr int kSubWindowMaxT = 32;
cudaError_t launch_decode(const LayerDev& L, const uint16_t* x, int T, const int32_t* ids,
                          const float* w, uint16_t* y, uint32_t flags, char* ws, const WsLayout& lay,
                          cudaStream_t st);
cudaError_t launch_prefill(const LayerDev& L, const uint16_t* x, int T, const int32_t* ids,
                           const float* w, uint16_t* y, int32_t* offsets_out, int32_t* entries_out,
                           uint32_t flags, char* ws, const WsLayout& lay, cudaStream_t st);

// Launch helper: programmatic dependent launch attribute on.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int sm_count();

// MOE_OK when the current device is an sm_100 GPU (cached per device), else
// MOE_ERR_NO_DEVICE.
moe_status check_device();

// moe_block_forward with an option to zero the workspace control block on the
// stream (after validation, before the first kernel).
moe_status block_forward(const moe_layer* layer, const void* x_bf16, int32_t T, void* y_bf16,
                         uint32_t flags, void* ws, size_t ws_bytes, void* stream,
                         bool clear_control);

}  // namespace moe
