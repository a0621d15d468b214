// meta_refresh.cuh -- the metadata of one page rebuilt by one thread block (EntmaxKV technical
// summary, §2.A: the bounding box kmin/kmax and the Gaussian statistics mean/variance of a
// page's keys). Used by the short-append metadata kernel and by the scan that refreshes the
// appended pages itself, so that both write the same bits.
#pragma once
#include "ekv_device.cuh"

namespace ekv {

// Clamped append range [s, s + n) of sequence b (len: its validated length). A range that
// starts before 0, ends past len or is longer than max_new is clamped and, when `report`,
// flags EKV_DEV_BAD_RANGE. Returns false when nothing is left to refresh.
__device__ __forceinline__ bool append_range(const ekv_cache &c, const int32_t *new_start,
                                             const int32_t *new_count, int max_new, int b,
                                             int len, bool report, int &s, int &n)
{
    s = new_start[b];
    n = new_count[b];
    if (n <= 0) return false;
    if (s < 0 || s + n > len || n > max_new) {
        if (report) flag(c.dev_status, EKV_DEV_BAD_RANGE);
        s = s < 0 ? 0 : (s > len ? len : s);
        const int e = s + n > len ? len : s + n;
        n = e - s > max_new ? max_new : e - s;
        if (n <= 0) return false;
    }
    return true;
}

template <int D>
struct MetaPageShared {
    float a[8][D], b[8][D], c[8][D];
    float mean[D];
};

// Page p of sequence b (length len), KV head h, by a block of 8 warps: warp w takes rows w,
// w + 8, ... (at most 8 each, P <= 64) with every load in flight and keeps them in registers for
// the variance pass; the warps' partial min / max / sums are combined in shared memory. A
// page-table entry outside [0, num_blocks) flags EKV_DEV_BAD_BLOCK and writes nothing. Every
// thread of the block must call it.
template <int DT, int D>
__device__ __forceinline__ void meta_refresh_page(const ekv_cache &c, int b, int h, int p, int len,
                                                  MetaPageShared<D> &sm)
{
    constexpr int VEC = D / 32;
    constexpr int RPW = 8;  // rows per warp: P <= 64 = 8 warps x 8 rows
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int P = c.page_size;
    const int blk = c.page_table[(size_t)b * c.max_pages + p];
    if (blk < 0 || blk >= c.num_blocks) {
        if (threadIdx.x == 0) flag(c.dev_status, EKV_DEV_BAD_BLOCK);
        return;
    }
    const int cnt = len - p * P < P ? len - p * P : P;
    const size_t row0 = ((size_t)blk * c.num_kv_heads + h) * P;
    const char *krow = static_cast<const char *>(c.k_cache) +
                       (row0 * D + lane * VEC) * (size_t)Chunk<DT>::kBytes;
    constexpr size_t ROWB = (size_t)D * Chunk<DT>::kBytes;
    float x[RPW][VEC];
#pragma unroll
    for (int u = 0; u < RPW; ++u)
        if (warp + 8 * u < cnt) load_vec_nc<DT, VEC>(krow + (warp + 8 * u) * ROWB, x[u]);
    float mn[VEC], mx[VEC], sum[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) { mn[e] = INFINITY; mx[e] = -INFINITY; sum[e] = 0.f; }
#pragma unroll
    for (int u = 0; u < RPW; ++u) {
        if (warp + 8 * u >= cnt) break;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            mn[e] = fminf(mn[e], x[u][e]);
            mx[e] = fmaxf(mx[e], x[u][e]);
            sum[e] += x[u][e];
        }
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        sm.a[warp][lane * VEC + e] = mn[e];
        sm.b[warp][lane * VEC + e] = mx[e];
        sm.c[warp][lane * VEC + e] = sum[e];
    }
    __syncthreads();
    const size_t mbase = ((size_t)blk * c.num_kv_heads + h) * 2 * D;
    for (int i = threadIdx.x; i < D; i += 256) {
        float lo = sm.a[0][i], hi = sm.b[0][i], s = sm.c[0][i];
#pragma unroll
        for (int w = 1; w < 8; ++w) {
            lo = fminf(lo, sm.a[w][i]);
            hi = fmaxf(hi, sm.b[w][i]);
            s += sm.c[w][i];
        }
        store_exact<DT>(c.meta_bbox, mbase + i, lo);
        store_exact<DT>(c.meta_bbox, mbase + D + i, hi);
        sm.mean[i] = s / (float)cnt;
    }
    if (!c.meta_mom) {
        __syncthreads();  // the block's partials may be overwritten by a next page
        return;
    }
    __syncthreads();
    float ss[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) ss[e] = 0.f;
#pragma unroll
    for (int u = 0; u < RPW; ++u) {
        if (warp + 8 * u >= cnt) break;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            const float dv = x[u][e] - sm.mean[lane * VEC + e];
            ss[e] = fmaf(dv, dv, ss[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) sm.a[warp][lane * VEC + e] = ss[e];
    __syncthreads();
    for (int i = threadIdx.x; i < D; i += 256) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += sm.a[w][i];
        c.meta_mom[mbase + i] = sm.mean[i];
        c.meta_mom[mbase + D + i] = v / (float)cnt;
    }
    __syncthreads();
}

}  // namespace ekv
