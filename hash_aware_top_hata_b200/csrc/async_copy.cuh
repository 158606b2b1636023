// async_copy.cuh -- inline-PTX wrappers for the sm_100a asynchronous
// global -> shared copies (cp.async, LSU path) that the HATA kernels stage
// their inputs with, plus the shared-memory address conversion they need.
#pragma once

#include <stdint.h>

namespace hata {

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Asynchronous 16-byte global -> shared copy.  No "memory" clobber:
// ordinary loads may move across it; the shared-memory data is only read
// after cp_async_wait (which does clobber) and a barrier.
__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src));
}
// The same with a source size of 0 or 16 bytes: 0 fills the 16 destination
// bytes with zeros and reads no global memory.
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src, uint32_t bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes));
}
// 4-, 8- or 16-byte copies (cache-all path; the 16-byte form above bypasses
// L1), source size 0 or N: 0 zero-fills the N destination bytes.
template <int N>
__device__ __forceinline__ void cp_async_zfill(uint32_t dst, const void *src, uint32_t bytes)
{
    static_assert(N == 4 || N == 8 || N == 16, "cp.async copies 4, 8 or 16 bytes");
    if constexpr (N == 16)
        cp_async16_zfill(dst, src, bytes);
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(dst), "l"(src), "n"(N),
                     "r"(bytes));
}
// The same copies with the whole source read (no zero fill).
template <int N>
__device__ __forceinline__ void cp_async_n(uint32_t dst, const void *src)
{
    static_assert(N == 4 || N == 8 || N == 16, "cp.async copies 4, 8 or 16 bytes");
    if constexpr (N == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src));
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst), "l"(src), "n"(N));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed cp.async groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace hata
