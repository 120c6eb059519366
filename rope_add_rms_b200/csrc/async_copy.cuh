// async_copy.cuh -- per-thread asynchronous global -> shared copies (cp.async, 16 bytes,
// cached in L2 only), in commit groups that a thread waits for in order.  Used to keep rows
// in flight in shared memory instead of registers.
#pragma once

#include <cstdint>

namespace nvn {

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace nvn

