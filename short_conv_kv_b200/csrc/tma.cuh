// Shared-memory barriers and bulk asynchronous copies (sm_90+ PTX, used on
// sm_100a): the pieces of a producer/consumer pipeline that streams rows
// from global memory into a shared-memory ring through the TMA unit.
//
// Every wait here is bounded in time: a waiter gives up after `timeout_ns`
// (read from %globaltimer) or as soon as another thread of the CTA has given
// up, so a logic error can never leave a CTA spinning forever.
#pragma once
#include <stdint.h>

namespace sconv {

// After a wait has given up, the copies already issued are still allowed to
// land (the CTA's shared memory must outlive them): this drain is bounded
// by its own fixed limit, whatever limit the pipeline waits were given.
constexpr unsigned long long kDrainTimeoutNs = 1000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Returns
// false (and raises *abort) on timeout; returns false soon after another
// thread has raised *abort.  The clock and the abort flag are checked once
// per 8 polls (each poll may suspend the thread for a while in hardware),
// so a waiting warp takes few issue slots from the warps that compute.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
#pragma unroll
    for (int i = 0; i < 8; ++i)  // unrolled: no counter register
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > timeout_ns) {
      *abort = 1;
      return false;
    }
  }
}

// Programmatic dependent launch: wait until the grids this one depends on
// have completed and their memory is visible (a no-op when the launch has
// no programmatic dependency).  Must precede every global-memory access.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Let the next grid in the stream start launching (its CTAs still wait in
// grid_dependency_wait() until this grid has completed).
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// One bulk copy global -> this CTA's shared memory, completion signalled on
// `bar` as transaction bytes.  dst, src 16-byte aligned; bytes % 16 == 0.
// (Plain load: no cluster multicast.)  The copy carries an L2 evict-first
// policy: the kernels read every input row exactly once, so the next reads
// should replace these lines rather than the cache rows just written
// (measured on B200: 8192-token prefill 18.4 -> 17.0 us, ring-state decode
// 7.7 -> 7.0 us; launches larger than L2 about 1 % slower).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 pol;\n\t"
      "createpolicy.fractional.L2::evict_first.b64 pol, 1.0;\n\t"
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], pol;\n\t}" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace sconv
