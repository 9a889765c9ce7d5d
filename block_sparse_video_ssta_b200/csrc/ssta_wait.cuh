// mbarrier primitives and the bounded waits used by every pipelined kernel of the
// library (and by the wait self-test, which exercises exactly this code).
//
// A wait never spins forever: after `timeout_ns` of global time without the phase
// completing, it records SSTA_ERR_DEVICE_TIMEOUT in the status word, raises the
// CTA's abort flag (which every other wait of the CTA watches) and returns false.
#pragma once

#include <stdint.h>

#include "ssta_internal.h"

namespace ssta {
namespace wait {
namespace {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct Ctl {
  volatile int* abort_flag;   // CTA-wide, in shared memory
  int32_t* status;            // device status word
  uint64_t timeout_ns;        // limit of one wait
};

// Polling loop of a bounded wait, entered only when the first try_wait gave up.  Kept
// out of line: a call costs a few hundred clocks (the caller's live registers go to the
// stack), which is why the first try sits inline in wait_bounded.
__device__ __noinline__ bool wait_bounded_slow(uint32_t bar, uint32_t parity, const Ctl& c) {
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*c.abort_flag) return false;
    if (global_ns() - t0 > c.timeout_ns) {
      *c.abort_flag = 1;
      atomicExch(c.status, (int)SSTA_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}
// Bounded wait by one thread: one inline try_wait (which itself blocks in hardware for a
// while and returns as soon as the phase completes), then the polling loop.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const Ctl& c) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_bounded_slow(bar, parity, c);
}
// Bounded wait by a whole warp; the outcome is made warp-uniform.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, const Ctl& c) {
  const bool ok = wait_bounded(bar, parity, c);
  return __all_sync(0xffffffffu, ok);
}
// Wait used while draining after an abort: bounded, never raises the flag.
__device__ __noinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > timeout_ns) return;
  }
}

}  // namespace
}  // namespace wait
}  // namespace ssta
