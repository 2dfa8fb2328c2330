// Helpers for the tcgen05 (5th-generation tensor core) kernels on sm_100a: tensor-memory
// allocation, TF32 MMA issue and completion, shared-memory matrix descriptors, proxy fences,
// named barriers, and the K-major 128-byte-swizzled operand rows.  Hand-written PTX.
#pragma once

#include "dw_internal.h"

namespace dwk {

// ---------------------------------------------------------------- PTX wrappers (sm_100a)
__device__ __forceinline__ void named_bar(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Named barrier that also ANDs a flag over the participating threads, so that a group of
// warps takes a give-up decision together (a warp that left alone would strand the others at
// their next barrier).
__device__ __forceinline__ bool named_bar_and(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(v ? 1u : 0u), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major, TF32 in, float32 accumulate.
__device__ __forceinline__ void mma_tf32(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on bar when every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128 bytes in groups of
// 8 rows (1024 bytes apart).  The leading-byte offset is unused in this mode.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = static_cast<uint64_t>((saddr & 0x3ffffu) >> 4);
    d |= static_cast<uint64_t>(1) << 16;              // leading byte offset (16 B, ignored)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;      // stride byte offset: next 8-row group
    d |= static_cast<uint64_t>(1) << 46;              // descriptor version for sm_100
    d |= static_cast<uint64_t>(2) << 61;              // 128-byte swizzle
    return d;
}

// ---------------------------------------------------------------- operand rows
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }

// Row `row` of a K-major 128-byte-swizzled tile: 16-byte chunk k lands at chunk k ^ (row % 8).
__device__ __forceinline__ void store_k_row(unsigned char *tile, int row, const float4 (&w)[8]) {
    unsigned char *base = tile + row * 128;  // 128-byte rows (32 TF32 words)
#pragma unroll
    for (int k = 0; k < 8; ++k) *reinterpret_cast<float4 *>(base + ((k ^ (row & 7)) << 4)) = w[k];
}

}  // namespace dwk
