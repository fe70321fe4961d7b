// cp_async.cuh -- asynchronous global -> shared copies (cp.async, sm_80+),
// used by the kernels that stage tiles while the previous tile computes.
#pragma once

#include "common.cuh"

namespace selscan {

// 16-byte asynchronous copy global -> shared (L2 only) of the first `bytes`
// (0..16) bytes of src; the rest of the 16 is zero-filled.  Both addresses
// 16-byte aligned.
__device__ __forceinline__ void cp_async16_n(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(bytes)
                 : "memory");
}
// The same with all 16 bytes copied when `valid`, none otherwise.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    cp_async16_n(dst, src, valid ? 16u : 0u);
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

}  // namespace selscan
