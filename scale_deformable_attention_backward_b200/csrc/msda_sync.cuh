// msda_sync.cuh -- shared-memory mbarrier helpers of the warp-specialised
// kernels (sm_100a): producer warps fill a ring of shared-memory slots with
// cp.async copies and generic stores, consumer warps read them.
//
// Every wait is bounded: past kWaitNs of %globaltimer a waiting thread raises
// the CTA's stop flag (so the other role stops waiting too) and the library's
// device failure flag, and the kernel returns with its outputs incomplete.
// The protocols here cannot stall when the code is right; the bound keeps a
// mistake from hanging the GPU.
#pragma once

#include <cstdint>

namespace msda {

constexpr unsigned long long kWaitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned bar_addr(const uint64_t* bar) {
  return static_cast<unsigned>(__cvta_generic_to_shared(bar));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned done;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}"
      : "=r"(done)
      : "r"(bar_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Arrive (release semantics: this thread's earlier shared-memory stores are
// visible to a thread whose wait on the completed phase returns).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar_addr(bar)) : "memory");
}

// An arrival that happens once every cp.async this thread has issued so far
// has landed (counts as one of the barrier's expected arrivals).
__device__ __forceinline__ void mbar_arrive_cp_async(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar_addr(bar))
               : "memory");
}

// Waits for the completion of the phase of `bar` with parity `parity`.  False
// if the CTA was told to stop or the wait ran past kWaitNs (then the stop flag
// and *failed are raised).
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, unsigned parity, volatile int* stop,
                                             int* failed) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned polls = 1;; ++polls) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*stop) return false;
    if ((polls & 255u) == 0 && global_ns() - t0 > kWaitNs) {
      *stop = 1;
      atomicExch(failed, 1);
      return false;
    }
  }
}

// Named barrier over `threads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace msda
