// Asynchronous 16-byte copies global -> shared (cp.async, the L2-only .cg form) used by the
// time-parallel passes to stage published aggregates, maps and carries while other work
// runs. Kept apart from the tile-movement helpers of wkv_device.cuh.
#pragma once

#include <cstdint>

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

}  // namespace wkv
