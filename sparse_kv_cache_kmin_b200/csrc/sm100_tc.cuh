// sm100_tc.cuh -- Blackwell (sm_100a) tensor-core and tensor-memory-access primitives used by
// the decode kernels: tiled TMA loads with 128-byte swizzle, shared-memory matrix descriptors,
// tcgen05.mma with fp32 accumulators in tensor memory (TMEM), and TMEM allocation / loads.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "ekv_device.cuh"

namespace ekv {

// ---- TMA: one 2-D tile (box) of a tensor map into shared memory, completing on `bar`
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- shared-memory matrix descriptor of a K-major operand in the 128-byte swizzled layout:
// rows of 128 bytes (64 bf16 of K), 8-row swizzle atoms 1024 bytes apart. Fields: start
// address >> 4 (bits 0-13), leading byte offset >> 4 (16-29, unused for this layout),
// stride byte offset >> 4 (32-45), descriptor version 1 (46-47), layout 2 = 128B swizzle (61-63).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(const void *smem_ptr)
{
    const uint64_t addr = smem_addr(smem_ptr);
    return ((addr >> 4) & 0x3FFFull) | (1ull << 16) | ((1024ull >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// ---- descriptor of an MN-major operand in the 128-byte swizzled layout: each 128-byte row
// holds 64 consecutive bf16 of M (or N) for one K index, 8 K rows form a 1024-byte swizzle atom;
// atoms along K are 1024 bytes apart (stride byte offset) and 64-element blocks along M are
// `lbo_bytes` apart (leading byte offset).
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(const void *smem_ptr, uint32_t lbo_bytes)
{
    const uint64_t addr = smem_addr(smem_ptr);
    return ((addr >> 4) & 0x3FFFull) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           ((1024ull >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// ---- instruction descriptor of tcgen05.mma.kind::f16: bf16 A and B (K-major), fp32 D,
// M x N tile: D format (bits 4-5) = 1 (f32), A format (7-9) = 1 (bf16), B format (10-12) = 1,
// N >> 3 (17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t mma_idesc_bf16_f32(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// the same with A MN-major (bit 15)
__host__ __device__ constexpr uint32_t mma_idesc_bf16_f32_amn(int M, int N)
{
    return mma_idesc_bf16_f32(M, N) | (1u << 15);
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, bool accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

// arrive on `bar` once every tcgen05.mma issued so far by this thread has completed
__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---- TMEM allocation (one full warp), address written to shared memory
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(dst_smem)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---- TMEM -> registers: 32 lanes x N consecutive 32-bit columns (this warp's lane quadrant)
template <int N> __device__ __forceinline__ void tmem_ld_32x32b(uint32_t taddr, uint32_t (&r)[N]);
template <> __device__ __forceinline__ void tmem_ld_32x32b<1>(uint32_t taddr, uint32_t (&r)[1])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr) : "memory");
}
template <> __device__ __forceinline__ void tmem_ld_32x32b<2>(uint32_t taddr, uint32_t (&r)[2])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr) : "memory");
}
template <> __device__ __forceinline__ void tmem_ld_32x32b<4>(uint32_t taddr, uint32_t (&r)[4])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(taddr) : "memory");
}
template <> __device__ __forceinline__ void tmem_ld_32x32b<8>(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

}  // namespace ekv
