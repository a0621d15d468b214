// step.cu -- page scores and top-k page selection of a decode step in one launch, one
// thread-block cluster per (sequence, KV head) (EntmaxKV technical summary, §2.A and §2.B.1).
//
// Every (sequence, KV head) pair is independent through scoring and selection, so a cluster
// of C CTAs owns one pair and nothing waits for the whole grid between the two steps.
//
// Scan: CTA r of the cluster takes the r-th slice of the pair's pages and streams their bbox
// rows -- a warp takes 16 pages at a time and each lane loads its 16-byte piece of all 16 rows
// (16 loads in flight per lane, 16 warps per SM: the deepest of the load structures measured
// on this layout), and the sign split
// max(q kmin, q kmax) = q+ kmax + q- kmin collapses the group bound to
// S_j = scale (Q+ . kmax_j + Q- . kmin_j). The scores stay in the CTA's shared memory as
// order-preserving 32-bit keys (and go to global memory only if the caller asks for them).
//
// Select: an exact radix select over the cluster's distributed shared memory. Per pass (11,
// 11 and 10 bits of the key, most significant first) every CTA counts its keys that match the
// prefix found so far into 2048 bins; after a cluster barrier each thread sums its bins over
// all CTAs of the cluster (DSMEM loads), and a block scan finds the bin holding the k-th
// largest key. The passes stop as soon as that bin is taken whole. Keys equal to the final
// threshold are taken in ascending page order, across CTAs in rank order. Each CTA then
// writes its kept pages at its offset of the ascending selection.
#include "cluster.cuh"

namespace ekv {

constexpr int kStepThreads = 512;      // one CTA per SM; 16 warps x 16 rows in flight per lane
constexpr int kStepKeyCap = 8192;      // pages per CTA (keys in shared memory)
constexpr int kStepBins = 2048;

__device__ __forceinline__ uint32_t score_key(float x)
{
    if (x != x) return 0u;                  // NaN sorts below everything
    uint32_t u = __float_as_uint(x + 0.0f);  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct StepShared {
    int hist[kStepBins];
    int warp_tot[32];
    int w_above[32], w_tie[32];  // per warp (the first NW entries)
    int s_bin, s_above, s_binc;
    int s_cnt[2];  // this CTA's (keys above the threshold, keys equal to it): read by the cluster
};

template <int DT, int D, int G>
__global__ void __launch_bounds__(kStepThreads, 1)
step_score_select_kernel(ekv_cache c, const void *__restrict__ q, int H_q, float scale, int topk,
                         float *__restrict__ scores, int32_t *__restrict__ sel_idx,
                         int32_t *__restrict__ sel_count, int max_sel)
{
    constexpr int NT = kStepThreads, NW = NT / 32;
    constexpr int BPT = kStepBins / NT;                    // histogram bins per thread
    constexpr int EPC = Chunk<DT>::N;
    constexpr int CPR = 2 * D * Chunk<DT>::kBytes / 16;  // 16-byte chunks per bbox row
    constexpr int W = CPR < 32 ? CPR : 32;                 // lanes per row
    constexpr int LPL = CPR / W;                           // chunks per lane per row
    constexpr int RPI = 32 / W;                            // rows per warp instruction
    constexpr int PG8 = 8;                                 // pages per reduction (as the standalone scan)
    constexpr int U = 2;                                   // reductions per warp step
    constexpr int PG = PG8 * U;                            // pages per warp step
    constexpr int NPL = PG8 / RPI;                         // page slots per lane per reduction
    extern __shared__ uint32_t keys[];                     // [kStepKeyCap]
    __shared__ StepShared sh;

    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_rank(), C = cluster_size();
    const int H = c.num_kv_heads, P = c.page_size;
    const int bh = blockIdx.x / (int)C, b = bh / H, h = bh % H;
    const int n = seq_pages(c.seq_lens, b, P, c.max_pages, (h == 0 && rank == 0) ? c.dev_status : nullptr,
                            nullptr);
    const int kk = topk < n ? topk : n;
    // this CTA's slice of the pages: whole PG-page groups
    const int ng = (n + PG - 1) / PG;
    const int p0 = (int)((long long)ng * rank / C) * PG;
    const int p1 = min((int)((long long)ng * (rank + 1) / C) * PG, n);
    const int nl = p1 > p0 ? p1 - p0 : 0;
    int32_t *out = sel_idx + (size_t)bh * max_sel;

    // ---------------------------------------------------------------- scan
    {
        float coef[LPL][EPC];
#pragma unroll
        for (int k = 0; k < LPL; ++k) {
            const int ci = k * W + lane % W;
            const bool upper = ci >= CPR / 2;
            const int cb = (ci % (CPR / 2)) * EPC;
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                float a = 0.f;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float qv = load_elem<DT>(q, ((size_t)b * H_q + h * G + g) * D + cb + e);
                    a += upper ? fmaxf(qv, 0.f) : fminf(qv, 0.f);
                }
                coef[k][e] = a;
            }
        }
        const char *bbox = static_cast<const char *>(c.meta_bbox);
        const int32_t *ptab = c.page_table + (size_t)b * c.max_pages;
        auto fetch_blk = [&](int gl) {  // block of page p0 + gl * PG + lane % PG; -1 past the slice, -2 bad
            int blk = -1;
            const int j = p0 + gl * PG + (lane & (PG - 1));
            if (j < p1) {
                blk = ptab[j];
                if (blk < 0 || blk >= c.num_blocks) {
                    flag(c.dev_status, EKV_DEV_BAD_BLOCK);
                    blk = -2;
                }
            }
            return blk;
        };
        const int ngl = (nl + PG - 1) / PG;
        int nblk = warp < ngl ? fetch_blk(warp) : -1;
        for (int gl = warp; gl < ngl; gl += NW) {
            const int myblk = nblk;
            uint4 x[U][NPL][LPL];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < NPL; ++i) {
                    const int blk = __shfl_sync(kFull, myblk, u * PG8 + i * RPI + lane / W);
#pragma unroll
                    for (int k = 0; k < LPL; ++k)
                        x[u][i][k] = blk >= 0 ? ld_stream16(bbox + (((size_t)blk * H + h) * CPR + k * W + lane % W) * 16)
                                              : make_uint4(0, 0, 0, 0);
                }
            if (gl + NW < ngl) nblk = fetch_blk(gl + NW);
            // per 8 pages, the standalone scan's arithmetic and reduction tree (identical scores)
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float part[NPL];
#pragma unroll
                for (int i = 0; i < NPL; ++i) {
                    part[i] = 0.f;
#pragma unroll
                    for (int k = 0; k < LPL; ++k) {
                        float f[EPC];
                        Chunk<DT>::unpack(x[u][i][k], f);
#pragma unroll
                        for (int e = 0; e < EPC; ++e) part[i] = fmaf(coef[k][e], f[e], part[i]);
                    }
                }
                transpose_reduce<NPL, W>(part, lane);
                const int po = transpose_index<NPL, W>(lane, 0) * RPI + lane / W;
                const int blk = __shfl_sync(kFull, myblk, u * PG8 + po);
                const int jl = gl * PG + u * PG8 + po;
                if (((lane % W) % (W / NPL)) == 0 && jl < nl) {
                    const float sc = blk >= 0 ? scale * part[0] : -INFINITY;
                    keys[jl] = score_key(sc);
                    if (scores) scores[(size_t)bh * c.max_pages + p0 + jl] = sc;
                }
            }
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- select
    if (kk == n) {  // every page is kept (also n = 0); p0 + nl <= n <= max_sel
        for (int i = tid; i < nl; i += NT) out[p0 + i] = p0 + i;
        if (rank == C - 1)
            for (int i = n + tid; i < max_sel; i += NT) out[i] = -1;
        if (rank == 0 && tid == 0) sel_count[bh] = n;
        pdl_trigger();
        return;
    }
    uint32_t prefix = 0, mask = 0;
    int remaining = kk;  // keys still to take among those matching the prefix
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int i = tid; i < kStepBins; i += NT) sh.hist[i] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < nl; i0 += NT) {
            const int i = i0 + tid;
            int bin = -1;
            if (i < nl) {
                const uint32_t u = keys[i];
                if ((u & mask) == prefix) bin = (int)((u >> shift) & (uint32_t)(nb - 1));
            }
            const unsigned peers = __match_any_sync(kFull, bin);
            if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], __popc(peers));
        }
        cluster_sync();
        // thread t owns bins nb-1-BPT*t ... nb-BPT-BPT*t (descending); sums over the cluster
        int cnt[BPT], sum = 0;
#pragma unroll
        for (int r = 0; r < BPT; ++r) {
            const int bin = nb - 1 - BPT * tid - r;
            cnt[r] = 0;
            if (bin >= 0)
                for (uint32_t cr = 0; cr < C; ++cr) cnt[r] += ld_dsmem(dsmem(&sh.hist[bin], cr));
            sum += cnt[r];
        }
        const int incl = block_incl_scan<NT>(sum, sh.warp_tot, nullptr);
        int run = incl - sum;
#pragma unroll
        for (int r = 0; r < BPT; ++r) {
            if (cnt[r] > 0 && run < remaining && remaining <= run + cnt[r]) {
                sh.s_bin = nb - 1 - BPT * tid - r;
                sh.s_above = run;
                sh.s_binc = cnt[r];
            }
            run += cnt[r];
        }
        cluster_sync();  // every CTA has read this pass's bins before any CTA clears them
        remaining -= sh.s_above;
        prefix |= (uint32_t)sh.s_bin << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        if (remaining == sh.s_binc) break;  // the bin is taken whole: lower bits cannot matter
    }
    // Kept: keys above the threshold T = prefix (on the masked bits), and the first `remaining`
    // keys equal to it in page order. Per warp, a contiguous range of this CTA's keys.
    const uint32_t T = prefix;
    auto cmp = [&](uint32_t u) -> int { const uint32_t um = u & mask; return um > T ? 1 : (um == T ? 0 : -1); };
    const int per = (nl + NW - 1) / NW;
    const int j0 = min(warp * per, nl), j1 = min(j0 + per, nl);
    int n_above = 0, n_tie = 0;
    for (int j = j0 + lane; j - lane < j1; j += 32) {
        const int cv = j < j1 ? cmp(keys[j]) : -1;
        n_above += __popc(__ballot_sync(kFull, cv > 0));
        n_tie += __popc(__ballot_sync(kFull, cv == 0));
    }
    if (lane == 0) { sh.w_above[warp] = n_above; sh.w_tie[warp] = n_tie; }
    __syncthreads();
    if (warp == 0) {
        const int a = lane < NW ? sh.w_above[lane] : 0, t = lane < NW ? sh.w_tie[lane] : 0;
        const int ia = warp_incl_scan(a), it = warp_incl_scan(t);
        sh.w_above[lane] = ia - a;  // above-keys before this warp
        sh.w_tie[lane] = it - t;    // ties before this warp
        if (lane == 31) { sh.s_cnt[0] = ia; sh.s_cnt[1] = it; }
    }
    cluster_sync();
    // this CTA's offset in the selection and the ties it takes: ties go in page order, and the
    // CTAs' slices are in rank order
    int off = 0, ties_before = 0;
    for (uint32_t cr = 0; cr < rank; ++cr) {
        const int a = ld_dsmem(dsmem(&sh.s_cnt[0], cr)), t = ld_dsmem(dsmem(&sh.s_cnt[1], cr));
        const int take = min(max(remaining - ties_before, 0), t);
        off += a + take;
        ties_before += t;
    }
    const int my_take = min(max(remaining - ties_before, 0), sh.s_cnt[1]);
    int tie_rank = sh.w_tie[warp];
    int pos = off + sh.w_above[warp] + min(tie_rank, my_take);
    for (int j = j0 + lane; j - lane < j1; j += 32) {
        const int cv = j < j1 ? cmp(keys[j]) : -1;
        const unsigned tb = __ballot_sync(kFull, cv == 0);
        const bool keep = cv > 0 || (cv == 0 && tie_rank + __popc(tb & ((1u << lane) - 1u)) < my_take);
        const unsigned kb = __ballot_sync(kFull, keep);
        const int at = pos + __popc(kb & ((1u << lane) - 1u));
        if (keep && at < kk) out[at] = p0 + j;
        pos += __popc(kb);
        tie_rank += __popc(tb);
    }
    if (rank == C - 1)
        for (int i = kk + tid; i < max_sel; i += NT) out[i] = -1;
    if (rank == 0 && tid == 0) sel_count[bh] = kk;
    cluster_sync();  // no CTA leaves while another may still read its counts
    pdl_trigger();
}

// Cluster size for `pairs` (sequence, KV head) pairs of at most `max_pages` pages: the largest
// power of two up to 16 with pairs * C CTAs still resident at once (one per SM), and at least
// enough CTAs that a slice (whole 16-page groups) fits the key capacity. 0 when none fits.
static int step_cluster_size(int pairs, int max_pages, int sms)
{
    int C = 1;
    while (C < 16 && (long long)pairs * C * 2 <= sms) C *= 2;
    while (C <= 16 && ((long long)max_pages + 16 * C - 1) / (16 * C) * 16 > kStepKeyCap) C *= 2;
    return C <= 16 ? C : 0;
}

template <int DT, int D, int G>
static cudaError_t launch_step_t(const ekv_cache &c, const void *q, int H_q, float scale, int topk,
                                 float *scores, int32_t *sel_idx, int32_t *sel_count, int max_sel,
                                 cudaStream_t st, bool pdl)
{
    auto k = step_score_select_kernel<DT, D, G>;
    static bool attr_set = false;  // per instantiation
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kStepKeyCap * (int)sizeof(uint32_t));
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int pairs = c.batch * c.num_kv_heads;
    int C = step_cluster_size(pairs, c.max_pages, sms);
    if (C == 0) return cudaErrorInvalidValue;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(pairs * C));
    cfg.blockDim = dim3(kStepThreads);
    const int keys = ((c.max_pages + 16 * C - 1) / (16 * C)) * 16;
    cfg.dynamicSmemBytes = sizeof(uint32_t) * (size_t)(keys < kStepKeyCap ? keys : kStepKeyCap);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    // a smaller cluster when the GPU cannot hold every cluster of this size at once (clusters
    // must fit in one GPC); the key capacity bounds how small it may get
    for (;;) {
        int active = 0;
        if (cudaOccupancyMaxActiveClusters(&active, (const void *)k, &cfg) != cudaSuccess) active = 0;
        const int Cn = C / 2;
        const bool fits_smaller = Cn >= 1 && ((c.max_pages + 16 * Cn - 1) / (16 * Cn)) * 16 <= kStepKeyCap;
        if (active >= pairs || !fits_smaller) break;
        C = Cn;
        attr[0].val.clusterDim.x = C;
        cfg.gridDim = dim3((unsigned)(pairs * C));
        const int kc = ((c.max_pages + 16 * C - 1) / (16 * C)) * 16;
        cfg.dynamicSmemBytes = sizeof(uint32_t) * (size_t)kc;
    }
    return cudaLaunchKernelEx(&cfg, k, c, q, H_q, scale, topk, scores, sel_idx, sel_count, max_sel);
}

template <int DT, int D>
static cudaError_t launch_step_g(const ekv_cache &c, const void *q, int H_q, float scale, int topk,
                                 float *scores, int32_t *sel_idx, int32_t *sel_count, int max_sel,
                                 cudaStream_t st, bool pdl)
{
    switch (H_q / c.num_kv_heads) {
    case 1: return launch_step_t<DT, D, 1>(c, q, H_q, scale, topk, scores, sel_idx, sel_count, max_sel, st, pdl);
    case 2: return launch_step_t<DT, D, 2>(c, q, H_q, scale, topk, scores, sel_idx, sel_count, max_sel, st, pdl);
    case 4: return launch_step_t<DT, D, 4>(c, q, H_q, scale, topk, scores, sel_idx, sel_count, max_sel, st, pdl);
    default: return launch_step_t<DT, D, 8>(c, q, H_q, scale, topk, scores, sel_idx, sel_count, max_sel, st, pdl);
    }
}

// Whether the fused scan and select serve this geometry: bf16 metadata, and pages per CTA
// within the key capacity for some cluster size of at most 16.
bool step_score_select_supported(const ekv_cache &c)
{
    return c.dtype == EKV_BF16 && step_cluster_size(c.batch * c.num_kv_heads, c.max_pages, 148) != 0;
}

cudaError_t launch_step_score_select(const ekv_cache &c, const void *q, int H_q, float scale,
                                     int topk, float *scores, int32_t *sel_idx, int32_t *sel_count,
                                     int max_sel, cudaStream_t st, bool pdl)
{
    return c.head_dim == 128 ? launch_step_g<EKV_BF16, 128>(c, q, H_q, scale, topk, scores, sel_idx, sel_count, max_sel, st, pdl)
                             : launch_step_g<EKV_BF16, 64>(c, q, H_q, scale, topk, scores, sel_idx, sel_count, max_sel, st, pdl);
}

}  // namespace ekv
