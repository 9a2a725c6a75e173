// Helpers of the time-parallel passes, kept apart from the tile-movement helpers of
// wkv_device.cuh: asynchronous 16-byte copies global -> shared (cp.async, the L2-only .cg
// form) that stage published aggregates, maps and carries while other work runs, and an
// mbarrier wait that suspends the warp instead of spinning.
#pragma once

#include <cstdint>

#include "wkv_device.cuh"

namespace wkv {

// One 16-byte copy from global to shared memory through L2 only; both addresses 16-byte
// aligned.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
// Closes the group of copies issued so far by this thread.
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits for every copy group of this thread.
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }


// try_wait with a suspend-time hint: the warp is suspended until the phase completes or
// about `hint_ns` pass, instead of the short system-dependent window of the plain form.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity,
                                                   uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase for kernels whose warps wait out the whole latency of
// their tile loads (nothing else to do meanwhile): suspended rather than spinning, so the
// wait costs a handful of instructions and leaves the issue slots to the SM's other warps.
// The wall-time limit is checked between suspensions; on give-up the error word is
// flagged and the caller carries on (as mbar_wait).
__device__ __forceinline__ void mbar_wait_suspend(uint64_t* bar, uint32_t parity, unsigned* err) {
  constexpr uint32_t kHintNs = 20000;
  if (mbar_try_wait_hint(bar, parity, kHintNs)) return;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 8; ++i)
      if (mbar_try_wait_hint(bar, parity, kHintNs)) return;
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(err, kErrTimeout);
      return;
    }
  }
}

}  // namespace wkv
