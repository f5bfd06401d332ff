// common.cuh -- device helpers shared by the kernels of the routed-MoE library:
// inline-PTX wrappers (mbarrier, bulk async copy, mma.sync, griddepcontrol),
// bounded waits, number-format helpers, and the workspace control block.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace moe {

// ---------------------------------------------------------------- constants
constexpr int kGroup = 32;      // quantisation group along K
constexpr int kTileRows = 16;   // packed row tile
constexpr int kMaxDecodeT = 8;  // decode window (mma n = 8)

// device error word bits (workspace control block)
constexpr uint32_t kErrTimeout = 1u;      // a bounded wait ran out
constexpr uint32_t kErrRange = 2u;        // an id / slot / size outside its range
constexpr uint32_t kErrNonFinite = 4u;    // a non-finite value where finite is required

// Bounded waits give up after this many nanoseconds of %globaltimer, unless
// the control block carries a limit of its own.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

// Test switch (control block word debug_withhold, honoured only under
// MOE_F_DEBUG): thread 0 of CTA 0 of the prefill gate/up GEMM's epilogue skips
// its plain arrive on the first accumulator's "TMEM free" barrier, so that the
// MMA issuer's wait before the CTA's third work item runs out.
constexpr uint32_t kWithholdPrefillArrive = 1u;

// Workspace control block (first 256 bytes of every workspace).
struct Control {
  uint32_t err;            // OR of kErr* bits
  uint32_t router_done;    // CTAs of the small-T router that finished (self-resetting)
  uint32_t prefill_done;   // CTAs of the prefill bucketing pass that finished (self-resetting)
  uint32_t wait_limit_us;  // bounded-wait limit in microseconds; 0: kWaitLimitNs
  uint32_t err_where;      // first failing site (debug aid)
  uint32_t debug_withhold; // test switch (kWithhold*), 0: off
  uint32_t pad[58];
};
static_assert(sizeof(Control) == 256, "control block is 256 bytes");

// ------------------------------------------------------------------- timing
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_error(Control* ctl, uint32_t bits, uint32_t where) {
  if (ctl) {
    uint32_t old = atomicOr(&ctl->err, bits);
    if (old == 0) atomicExch(&ctl->err_where, where);
  }
}

// -------------------------------------------------------------- shared addr
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about `ns` nanoseconds pass, instead of spinning on the issue
// slots that the other warps of its SM sub-partition need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; gives up after the
// control block's limit (kWaitLimitNs when it holds 0) of %globaltimer,
// records kErrTimeout and returns false.  The limit is read only once a wait
// has lasted kWaitFloorNs, so the waits of a running pipeline never load it;
// limits below the floor are not accepted by the host.
constexpr unsigned long long kWaitFloorNs = 1000000ull;   // 1 ms
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Control* ctl,
                                          uint32_t where) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  unsigned long long limit = 0;   // not read yet
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
    const unsigned long long el = globaltimer_ns() - t0;
    if (el > kWaitFloorNs) {
      if (limit == 0) {
        const uint32_t us = ctl ? *reinterpret_cast<volatile uint32_t*>(&ctl->wait_limit_us) : 0u;
        limit = us ? 1000ull * us : kWaitLimitNs;
      }
      if (el > limit) {
        record_error(ctl, kErrTimeout, where);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------ bulk async copy
// global -> shared, completion signalled on an mbarrier (complete_tx).
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Hint: bring [src, src + bytes) into L2.  16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------------ programmatic dependent launch
// griddepcontrol.wait: block until the grids this one depends on completed and
// their memory is visible (a no-op when launched without the PDL attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next grid in the stream to start launching.  Every kernel here
// calls it only after its own pdl_wait(), so a dependent grid may read the
// outputs of the grid two launches back before its own wait.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// -------------------------------------------------------------- mma.sync
// D(16x8 f32) = A(16x16 f16, row) * B(16x8 f16, col) + C
// Not volatile: the compiler may interleave independent MMAs and their loads.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4],
                                              const uint32_t (&b)[2], const float (&c)[4]) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

// ------------------------------------------------------------ bit helpers
// (a & b) | c in one LOP3
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Orderable key of a float for "largest first": NaN lowest, -0 == +0.
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v != v) return 0u;
  uint32_t u = (v == 0.0f) ? 0u : __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Named barrier over `count` threads (multiple of 32).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier over `count` threads that also returns whether any of them
// passed pred = true (every participant gets the same answer).
__device__ __forceinline__ bool named_bar_any(uint32_t id, uint32_t count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

}  // namespace moe
