// quality.cu -- how much of the full-cache attention a page selection keeps (EntmaxKV technical
// summary, §3: attending over a subset of the tokens moves the output by at most 2 B delta,
// delta the full-cache weight outside the subset; §3-§4: whether the kept pages hold the
// support of the full-cache entmax). A diagnostic beside the decode, not a step of it: it reads
// every key of every sequence.
//
// One CTA per (slice of kQualPages pages, sequence x KV head). The kept pages of the slice are a
// bitmap in shared memory and the G query rows, pre-scaled, sit beside it. A warp takes token
// rows in turn, four at once (lane l owns elements l, l + 32, ...), and per query turns the
// logit into the full-cache weight the given statistic defines: softmax exp(s - LSE), entmax
// [z - tau]_+^(1/(alpha-1)) with z = (alpha-1) s. Weights of tokens outside the selection are
// summed in fp64 (delta); support members (entmax: z > tau; softmax: every valid token) are
// counted, in and out of the selection. CTA partials are added into the caller's outputs,
// which the entry point zeroes first.
#include "ekv_device.cuh"

namespace ekv {

constexpr int kQualPages = 256;  // pages per CTA
constexpr int kQualRows = 4;     // token rows in flight per warp

template <int DT, int D, int G>
__global__ void __launch_bounds__(256)
quality_kernel(ekv_cache c, const void *__restrict__ q, int H_q, float scale, int attn,
               const float *__restrict__ stat_full, const int32_t *__restrict__ sel_idx,
               const int32_t *__restrict__ sel_count, int max_sel, double *__restrict__ dropped,
               int32_t *__restrict__ support)
{
    __shared__ float qs[G][D];
    __shared__ uint32_t kept[kQualPages / 32];
    __shared__ double red_d[8][G];
    __shared__ int red_n[8][G][2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = c.num_kv_heads, P = c.page_size;
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    int len;
    const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
    const int p0 = blockIdx.x * kQualPages;
    if (p0 >= np) return;
    const int p1 = p0 + kQualPages < np ? p0 + kQualPages : np;
    for (int i = tid; i < G * D; i += 256)
        qs[i / D][i % D] = scale * load_elem<DT>(q, ((size_t)b * H_q + (size_t)h * G + i / D) * D + i % D);
    if (tid < kQualPages / 32) kept[tid] = 0u;
    __syncthreads();
    int ns = sel_count[bh];
    ns = ns < 0 ? 0 : (ns > max_sel ? max_sel : ns);
    for (int i = tid; i < ns; i += 256) {
        const int j = sel_idx[(size_t)bh * max_sel + i];
        if (j >= p0 && j < p1) atomicOr(&kept[(j - p0) >> 5], 1u << ((j - p0) & 31));
    }
    float st[G];
#pragma unroll
    for (int g = 0; g < G; ++g) st[g] = stat_full[(size_t)b * H_q + (size_t)h * G + g];
    const float am1 = attn == EKV_ENTMAX15 ? 0.5f : 1.0f;  // alpha - 1 (entmax modes)
    __syncthreads();

    double dsum[G];
    int nsup[G], nin[G];
#pragma unroll
    for (int g = 0; g < G; ++g) { dsum[g] = 0.0; nsup[g] = 0; nin[g] = 0; }
    const int t0 = p0 * P, t1 = (p1 * P < len ? p1 * P : len);
    for (int tb = t0 + warp * kQualRows; tb < t1; tb += 8 * kQualRows) {
        float kv[kQualRows][D / 32];
        int blk[kQualRows];
#pragma unroll
        for (int r = 0; r < kQualRows; ++r) {
            const int t = tb + r;
            blk[r] = -1;
            if (t < t1) {
                blk[r] = c.page_table[(size_t)b * c.max_pages + t / P];
                if (blk[r] < 0 || blk[r] >= c.num_blocks) {
                    if (lane == 0 && t % P == 0) flag(c.dev_status, EKV_DEV_BAD_BLOCK);
                    blk[r] = -1;
                }
            }
            const size_t row = ((size_t)(blk[r] < 0 ? 0 : blk[r]) * H + h) * P + t % P;
#pragma unroll
            for (int e = 0; e < D / 32; ++e)
                kv[r][e] = blk[r] >= 0 ? load_elem<DT>(c.k_cache, row * D + lane + 32 * e) : 0.f;
        }
#pragma unroll
        for (int r = 0; r < kQualRows; ++r) {
            if (blk[r] < 0) continue;  // uniform over the warp
            const int j = (tb + r) / P;
            const bool in = (kept[(j - p0) >> 5] >> ((j - p0) & 31)) & 1u;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < D / 32; ++e) s = fmaf(qs[g][lane + 32 * e], kv[r][e], s);
                s = warp_sum(s);
                float p;
                bool member;
                if (attn == EKV_SOFTMAX) {
                    p = expf(s - st[g]);
                    member = true;
                } else {
                    const float rr = am1 * s - st[g];
                    member = rr > 0.f;
                    p = member ? (attn == EKV_SPARSEMAX ? rr : rr * rr) : 0.f;
                }
                if (!in) dsum[g] += (double)p;
                nsup[g] += member;
                nin[g] += member && in;
            }
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            red_d[warp][g] = dsum[g];
            red_n[warp][g][0] = nsup[g];
            red_n[warp][g][1] = nin[g];
        }
    }
    __syncthreads();
    if (tid < G) {
        double dd = 0.0;
        int a = 0, k = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) { dd += red_d[w][tid]; a += red_n[w][tid][0]; k += red_n[w][tid][1]; }
        const size_t bq = (size_t)b * H_q + (size_t)h * G + tid;
        atomicAdd(dropped + bq, dd);
        atomicAdd(support + 2 * bq, a);
        atomicAdd(support + 2 * bq + 1, k);
    }
}

template <int DT, int D, int G>
static cudaError_t launch_quality_t(const ekv_cache &c, const void *q, int H_q, float scale,
                                    int attn, const float *stat_full, const int32_t *sel_idx,
                                    const int32_t *sel_count, int max_sel, double *dropped,
                                    int32_t *support, cudaStream_t st)
{
    const dim3 grid((c.max_pages + kQualPages - 1) / kQualPages, c.batch * c.num_kv_heads);
    quality_kernel<DT, D, G><<<grid, 256, 0, st>>>(c, q, H_q, scale, attn, stat_full, sel_idx,
                                                   sel_count, max_sel, dropped, support);
    return cudaGetLastError();
}

template <int DT, int D>
static cudaError_t launch_quality_g(const ekv_cache &c, const void *q, int H_q, float scale,
                                    int attn, const float *stat_full, const int32_t *sel_idx,
                                    const int32_t *sel_count, int max_sel, double *dropped,
                                    int32_t *support, cudaStream_t st)
{
    switch (H_q / c.num_kv_heads) {
    case 1: return launch_quality_t<DT, D, 1>(c, q, H_q, scale, attn, stat_full, sel_idx, sel_count, max_sel, dropped, support, st);
    case 2: return launch_quality_t<DT, D, 2>(c, q, H_q, scale, attn, stat_full, sel_idx, sel_count, max_sel, dropped, support, st);
    case 4: return launch_quality_t<DT, D, 4>(c, q, H_q, scale, attn, stat_full, sel_idx, sel_count, max_sel, dropped, support, st);
    default: return launch_quality_t<DT, D, 8>(c, q, H_q, scale, attn, stat_full, sel_idx, sel_count, max_sel, dropped, support, st);
    }
}

cudaError_t launch_selection_quality(const ekv_cache &c, const void *q, int H_q, float scale,
                                     int attn, const float *stat_full, const int32_t *sel_idx,
                                     const int32_t *sel_count, int max_sel, double *dropped,
                                     int32_t *support, cudaStream_t st)
{
    cudaError_t e = cudaMemsetAsync(dropped, 0, sizeof(double) * (size_t)c.batch * H_q, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(support, 0, sizeof(int32_t) * 2 * (size_t)c.batch * H_q, st);
    if (e != cudaSuccess) return e;
    if (c.dtype == EKV_BF16)
        return c.head_dim == 128 ? launch_quality_g<EKV_BF16, 128>(c, q, H_q, scale, attn, stat_full, sel_idx, sel_count, max_sel, dropped, support, st)
                                 : launch_quality_g<EKV_BF16, 64>(c, q, H_q, scale, attn, stat_full, sel_idx, sel_count, max_sel, dropped, support, st);
    return c.head_dim == 128 ? launch_quality_g<EKV_F32, 128>(c, q, H_q, scale, attn, stat_full, sel_idx, sel_count, max_sel, dropped, support, st)
                             : launch_quality_g<EKV_F32, 64>(c, q, H_q, scale, attn, stat_full, sel_idx, sel_count, max_sel, dropped, support, st);
}

}  // namespace ekv
