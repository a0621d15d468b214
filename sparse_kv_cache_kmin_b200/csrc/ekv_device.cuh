// ekv_device.cuh -- device helpers shared by the sm_100a kernels of libekv.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ekv.h"

namespace ekv {

constexpr unsigned kFull = 0xffffffffu;

// 16-byte streaming load through the non-coherent path: no L1 allocation (every byte is
// used once by the warp that loads it), 256-byte L2 prefetch (metadata rows and page spans
// are >= 256 contiguous bytes).
__device__ __forceinline__ uint4 ld_stream16(const void *p)
{
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}
// 16 bytes through L2 only: for data the same kernel wrote (ordered by a barrier before it)
__device__ __forceinline__ uint4 ld_cg16(const void *p)
{
    uint4 r;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p)
                 : "memory");
    return r;
}

// A 16-byte chunk of stored elements, widened to fp32. bf16 is the upper half of an IEEE
// float32, so widening is a shift; the element at the lower address is the low half.
template <int DT> struct Chunk;

template <> struct Chunk<EKV_BF16> {
    static constexpr int N = 8;
    static constexpr int kBytes = 2;
    __device__ __forceinline__ static void unpack(const uint4 &w, float (&f)[8])
    {
        f[0] = __uint_as_float(w.x << 16); f[1] = __uint_as_float(w.x & 0xffff0000u);
        f[2] = __uint_as_float(w.y << 16); f[3] = __uint_as_float(w.y & 0xffff0000u);
        f[4] = __uint_as_float(w.z << 16); f[5] = __uint_as_float(w.z & 0xffff0000u);
        f[6] = __uint_as_float(w.w << 16); f[7] = __uint_as_float(w.w & 0xffff0000u);
    }
};

template <> struct Chunk<EKV_F32> {
    static constexpr int N = 4;
    static constexpr int kBytes = 4;
    __device__ __forceinline__ static void unpack(const uint4 &w, float (&f)[4])
    {
        f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
        f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
    }
};

// Element load / store in the cache dtype.
template <int DT> __device__ __forceinline__ float load_elem(const void *p, size_t i);
template <> __device__ __forceinline__ float load_elem<EKV_F32>(const void *p, size_t i)
{
    return static_cast<const float *>(p)[i];
}
template <> __device__ __forceinline__ float load_elem<EKV_BF16>(const void *p, size_t i)
{
    return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t *>(p)[i]) << 16);
}

// Store a value that is exactly representable in the dtype (a min or max of stored values).
template <int DT> __device__ __forceinline__ void store_exact(void *p, size_t i, float v);
template <> __device__ __forceinline__ void store_exact<EKV_F32>(void *p, size_t i, float v)
{
    static_cast<float *>(p)[i] = v;
}
template <> __device__ __forceinline__ void store_exact<EKV_BF16>(void *p, size_t i, float v)
{
    static_cast<uint16_t *>(p)[i] = static_cast<uint16_t>(__float_as_uint(v) >> 16);
}

// Reduce N per-lane values across each aligned group of W lanes (W a power of two dividing
// 32, N a power of two) with a transposing butterfly: at every step a lane keeps half of its
// values and ships the other half to its partner, so the N sums cost about N + log2(W)
// shuffles instead of N * log2(W). On return v[0 .. max(N / W, 1)) hold complete sums; value
// slot r of lane l is original index r + sum over the halving steps s of
// bit(l, W >> (s + 1)) * (N >> (s + 1)), i.e. for N <= W lane l holds index (l % W) / (W / N).
template <int N, int W>
__device__ __forceinline__ void transpose_reduce(float (&v)[N], int lane)
{
    int n = N;
#pragma unroll
    for (int o = W / 2; o >= 1; o >>= 1) {
        if (n > 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                if (i < n / 2) {
                    float send = upper ? v[i] : v[i + n / 2];
                    float keep = upper ? v[i + n / 2] : v[i];
                    v[i] = keep + __shfl_xor_sync(kFull, send, o);
                }
            }
            n >>= 1;
        } else {
            v[0] += __shfl_xor_sync(kFull, v[0], o);
        }
    }
}

// Index of the value that lane `lane` holds in slot r after transpose_reduce<N, W>.
template <int N, int W>
__device__ __forceinline__ int transpose_index(int lane, int r)
{
    int idx = r, n = N;
#pragma unroll
    for (int o = W / 2; o >= 1 && n > 1; o >>= 1) {
        if (lane & o) idx += n / 2;
        n >>= 1;
    }
    return idx;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}
__device__ __forceinline__ int warp_sum(int v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

__device__ __forceinline__ void flag(uint32_t *status, uint32_t bit)
{
    if (status) atomicOr(status, bit);
}

// Pages of a sequence, with the length validated against the page-table row.
__device__ __forceinline__ int seq_pages(const int32_t *seq_lens, int b, int P, int max_pages,
                                         uint32_t *status, int *len_out)
{
    int len = seq_lens[b];
    if (len < 0 || len > max_pages * P) {
        flag(status, EKV_DEV_BAD_LEN);
        len = len < 0 ? 0 : max_pages * P;
    }
    if (len_out) *len_out = len;
    return (len + P - 1) / P;
}

}  // namespace ekv

namespace ekv {

// Inclusive scan of one int per thread over a block of NT threads (NT a multiple of 32).
// warp_tot: shared scratch of NT/32 ints. *total (if given) receives the block total.
// Contains __syncthreads(); every thread of the block must call it.
template <int NT>
__device__ __forceinline__ int block_incl_scan(int v, int *warp_tot, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NT / 32 ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(kFull, w, o);
            if (lane >= o) w += t;
        }
        if (lane < NT / 32) warp_tot[lane] = w;
    }
    __syncthreads();
    if (warp > 0) v += warp_tot[warp - 1];
    if (total) *total = warp_tot[NT / 32 - 1];
    __syncthreads();
    return v;
}

// Inclusive warp scan.
__device__ __forceinline__ int warp_incl_scan(int v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// Programmatic dependent launch: wait for the preceding grid in the stream (no-op when the
// launch did not opt in), then let the next grid be scheduled at once. Every libekv kernel
// waits here before it reads anything an earlier kernel wrote, so an early start only lets
// the next kernel's CTAs take SM slots as this grid's CTAs leave, instead of after the grid.
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
}
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;"); }

}  // namespace ekv

namespace ekv {

// Non-coherent load of VEC consecutive elements of dtype DT (VEC * size bytes, naturally
// aligned), widened to fp32.
template <int DT, int VEC>
__device__ __forceinline__ void load_vec_nc(const void *p, float (&f)[VEC])
{
    constexpr int BYTES = VEC * Chunk<DT>::kBytes;
    uint32_t w[4] = {0, 0, 0, 0};
    if constexpr (BYTES == 16) {
        asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
            : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "l"(p));
    } else if constexpr (BYTES == 8) {
        asm("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "l"(p));
    } else {
        static_assert(BYTES == 4, "4, 8 or 16 bytes");
        asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(w[0]) : "l"(p));
    }
    if constexpr (DT == EKV_BF16) {
#pragma unroll
        for (int i = 0; i < VEC / 2; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) f[i] = __uint_as_float(w[i]);
    }
}

// Persistent-grid size for a kernel: SM count x resident CTAs per SM, cached per
// (kernel, device, dynamic shared memory).
int persistent_grid_size(const void *kernel, int threads, size_t smem);

// Whether consecutive libekv kernels use programmatic dependent launch (environment variable
// EKV_PDL=0 turns it off for every entry point).
bool use_pdl();

}  // namespace ekv

namespace ekv {

// ---- shared-memory barriers and bulk (TMA) copies, sm_90+ PTX
__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// arrive (count 1) and add `bytes` to the transaction count of the current phase
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase of `parity` to complete, giving up after `limit_ns` nanoseconds.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t limit_ns = 2000000000ull)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > limit_ns) return false;
    return true;
}
// One bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16), its
// completion counted on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}
// Named barrier over the first `threads` threads of the block (id 1..15).
// Start moving a line towards L2 (no register result, no wait).
__device__ __forceinline__ void prefetch_l2(const void *p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ void named_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier that also ANDs a flag over the participating threads: every thread gets the
// same answer, so a group of warps leaves a loop together or not at all.
__device__ __forceinline__ bool named_sync_and(int id, int threads, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, %3, p;\n"
        " selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(threads)
        : "memory");
    return r != 0;
}

}  // namespace ekv
