// meta_update.cu -- per-page key metadata upkeep (EntmaxKV technical summary, §2.A: the
// bounding box kmin/kmax and the Gaussian statistics mean/variance of each page's keys,
// kept up to date as pages fill).
//
// Prefill and long appends: one warp per (touched page, KV head). A warp reads the page's
// valid key rows of its head (P rows of d elements, contiguous in the [block][head][P][d]
// layout) with lane l owning coordinates [l * d/32, (l+1) * d/32): min, max and sum in one
// pass, then the squared deviations from the fp32 mean in a second pass over the same rows
// (two-pass variance; the rows are still in L1/L2). kmin/kmax are stored in the cache dtype
// (exact: they are stored values); mean and population variance in fp32.
#include "ekv_device.cuh"
#include "meta_refresh.cuh"

namespace ekv {

template <int DT, int D>
__global__ void __launch_bounds__(256)
page_meta_update_kernel(ekv_cache c, const int32_t *__restrict__ new_start,
                        const int32_t *__restrict__ new_count, int max_new)
{
    pdl_wait();
    constexpr int VEC = D / 32;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.z * 8 + (threadIdx.x >> 5);
    const int b = blockIdx.y;
    const int P = c.page_size;
    if (h >= c.num_kv_heads) return;

    int len;
    seq_pages(c.seq_lens, b, P, c.max_pages, c.dev_status, &len);
    int s = new_start[b], n = new_count[b];
    if (n <= 0) return;
    if (s < 0 || s + n > len || n > max_new) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag(c.dev_status, EKV_DEV_BAD_RANGE);
        s = s < 0 ? 0 : (s > len ? len : s);
        int e = s + n > len ? len : s + n;
        n = e - s > max_new ? max_new : e - s;
        if (n <= 0) return;
    }
    const int p = s / P + blockIdx.x;
    if (p > (s + n - 1) / P) return;
    const int blk = c.page_table[(size_t)b * c.max_pages + p];
    if (blk < 0 || blk >= c.num_blocks) {
        if (lane == 0) flag(c.dev_status, EKV_DEV_BAD_BLOCK);
        return;
    }
    const int cnt = len - p * P < P ? len - p * P : P;
    const size_t row0 = ((size_t)blk * c.num_kv_heads + h) * P;

    // The page's rows are read 8 tokens at a time, each lane's VEC coordinates with one
    // vector load per token, so a warp keeps 8 loads in flight per lane instead of walking the
    // tokens one dependent load after another.
    constexpr int TB = 8;
    const char *krow = static_cast<const char *>(c.k_cache) +
                       (row0 * D + lane * VEC) * (size_t)Chunk<DT>::kBytes;
    constexpr size_t ROWB = (size_t)D * Chunk<DT>::kBytes;
    float mn[VEC], mx[VEC], sum[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) { mn[e] = INFINITY; mx[e] = -INFINITY; sum[e] = 0.f; }
    for (int t0 = 0; t0 < cnt; t0 += TB) {
        float x[TB][VEC];
#pragma unroll
        for (int u = 0; u < TB; ++u)
            if (t0 + u < cnt) load_vec_nc<DT, VEC>(krow + (t0 + u) * ROWB, x[u]);
#pragma unroll
        for (int u = 0; u < TB; ++u) {
            if (t0 + u >= cnt) break;
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                mn[e] = fminf(mn[e], x[u][e]);
                mx[e] = fmaxf(mx[e], x[u][e]);
                sum[e] += x[u][e];
            }
        }
    }
    const size_t mbase = ((size_t)blk * c.num_kv_heads + h) * 2 * D;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        store_exact<DT>(c.meta_bbox, mbase + lane * VEC + e, mn[e]);
        store_exact<DT>(c.meta_bbox, mbase + D + lane * VEC + e, mx[e]);
    }
    if (c.meta_mom) {
        float mean[VEC], ss[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) { mean[e] = sum[e] / (float)cnt; ss[e] = 0.f; }
        for (int t0 = 0; t0 < cnt; t0 += TB) {
            float x[TB][VEC];
#pragma unroll
            for (int u = 0; u < TB; ++u)
                if (t0 + u < cnt) load_vec_nc<DT, VEC>(krow + (t0 + u) * ROWB, x[u]);
#pragma unroll
            for (int u = 0; u < TB; ++u) {
                if (t0 + u >= cnt) break;
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float dv = x[u][e] - mean[e];
                    ss[e] = fmaf(dv, dv, ss[e]);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            c.meta_mom[mbase + lane * VEC + e] = mean[e];
            c.meta_mom[mbase + D + lane * VEC + e] = ss[e] / (float)cnt;
        }
    }
}

// The same statistics for a short append (a page or two per sequence per step): one CTA per
// (touched page, KV head), so the page's rows are read once, all at the same time
// (meta_refresh_page).
template <int DT, int D>
__global__ void __launch_bounds__(256)
page_meta_wide_kernel(ekv_cache c, const int32_t *__restrict__ new_start,
                      const int32_t *__restrict__ new_count, int max_new)
{
    __shared__ MetaPageShared<D> sm;
    pdl_wait();
    const int h = blockIdx.z, b = blockIdx.y;
    const int P = c.page_size;
    int len;
    seq_pages(c.seq_lens, b, P, c.max_pages, c.dev_status, &len);
    int s, n;
    if (!append_range(c, new_start, new_count, max_new, b, len,
                      blockIdx.x == 0 && h == 0 && threadIdx.x == 0, s, n))
        return;
    const int p = s / P + blockIdx.x;
    if (p > (s + n - 1) / P) return;
    meta_refresh_page<DT, D>(c, b, h, p, len, sm);
}

cudaError_t launch_page_meta_update(const ekv_cache &c, const int32_t *new_start,
                                    const int32_t *new_count, int max_new, cudaStream_t st)
{
    // A short append (at most two pages of tokens): one CTA per touched page and head.
    if (max_new > 0 && max_new <= 2 * c.page_size) {
        const dim3 gw((max_new + c.page_size - 1) / c.page_size + 1, c.batch, c.num_kv_heads);
#define EKV_META_W(DT, D) page_meta_wide_kernel<DT, D><<<gw, 256, 0, st>>>(c, new_start, new_count, max_new)
        if (c.dtype == EKV_BF16) {
            if (c.head_dim == 128) EKV_META_W(EKV_BF16, 128); else EKV_META_W(EKV_BF16, 64);
        } else {
            if (c.head_dim == 128) EKV_META_W(EKV_F32, 128); else EKV_META_W(EKV_F32, 64);
        }
#undef EKV_META_W
        return cudaGetLastError();
    }
    // A range of max_new tokens starting anywhere touches at most ceil(max_new / P) + 1 pages.
    const int P = c.page_size;
    dim3 grid((max_new + P - 1) / P + 1, c.batch, (c.num_kv_heads + 7) / 8);
    if (max_new == 0) return cudaSuccess;
#define EKV_META(DT, D) page_meta_update_kernel<DT, D><<<grid, 256, 0, st>>>(c, new_start, new_count, max_new)
    if (c.dtype == EKV_BF16) {
        if (c.head_dim == 128) EKV_META(EKV_BF16, 128); else EKV_META(EKV_BF16, 64);
    } else {
        if (c.head_dim == 128) EKV_META(EKV_F32, 128); else EKV_META(EKV_F32, 64);
    }
#undef EKV_META
    return cudaGetLastError();
}

// The device-side timeout path on its own: one thread waits on an mbarrier that nothing ever
// arrives on, with the bounded wait every pipelined kernel uses; when the limit runs out it sets
// EKV_DEV_TIMEOUT and the kernel returns. No copy is in flight, so giving up is always safe.
__global__ void wait_selftest_kernel(uint32_t *status, uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        if (!mbar_wait_bounded(&bar, 0, limit_ns)) flag(status, EKV_DEV_TIMEOUT);
    }
}

cudaError_t launch_wait_selftest(uint32_t *status, uint64_t limit_ns, cudaStream_t st)
{
    wait_selftest_kernel<<<1, 32, 0, st>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace ekv
