// score.cu -- query-aware page scoring from the page metadata only (EntmaxKV technical
// summary, §2.A), before any key or value is read.
//
// Top-k policy: the group bound S_j = sum_g scale * sum_c max(q_gc kmin_jc, q_gc kmax_jc).
// Because kmin <= kmax coordinate-wise, max(q kmin, q kmax) = q+ kmax + q- kmin with
// q+ = max(q, 0), q- = min(q, 0); summed over the group this is
//     S_j = scale * (Q+ . kmax_j + Q- . kmin_j),   Q+- = sum_g q_g+-,
// two FMAs per coordinate per page whatever the group size: the scan is bound by HBM.
//
// Layout and traffic: a page's bbox row for one KV head is 2*d contiguous elements (512 B for
// bf16 d=128). A warp streams whole rows with 16-byte loads (lane l owns the l-th 16 bytes,
// i.e. eight kmin or eight kmax coordinates, and holds the matching eight Q- or Q+
// coefficients in registers), eight pages per step so that each lane has eight independent
// loads in flight, then a transposing butterfly reduces the eight per-page partial dots in
// nine shuffles. The grid is persistent (a few CTAs per SM); the flattened work list of
// (sequence, KV head, 8-page group) is split evenly over CTAs, so ragged batches balance.
//
// Gaussian policy: per query, UB_gj (as above but unsummed), m_gj = scale * q_g . mean_j and
// v_gj = scale^2 * sum_c q_gc^2 var_jc; each page reads its bbox row and its fp32 moment row.
#include "ekv_device.cuh"
#include "meta_refresh.cuh"

namespace ekv {

// Prefix over sequences of the work groups each contributes: H_kv * ceil(n_pages / PG).
template <int PG>
__device__ __forceinline__ int build_group_prefix(const ekv_cache &c, int *pre, int *warp_tot)
{
    const int B = c.batch;
    int run = 0;
    for (int b0 = 0; b0 < B; b0 += 256) {
        const int b = b0 + (int)threadIdx.x;
        int v = 0;
        if (b < B) {
            int np = seq_pages(c.seq_lens, b, c.page_size, c.max_pages,
                               blockIdx.x == 0 ? c.dev_status : nullptr, nullptr);
            v = c.num_kv_heads * ((np + PG - 1) / PG);
        }
        int tot;
        int incl = block_incl_scan<256>(v, warp_tot, &tot);
        if (b < B) pre[b] = run + incl - v;
        run += tot;
    }
    if (threadIdx.x == 0) pre[B] = run;
    __syncthreads();
    return run;
}

// Largest b with pre[b] <= gi (pre non-decreasing, pre[0] = 0 <= gi < pre[B]).
__device__ __forceinline__ int find_seq(const int *pre, int B, long gi)
{
    int lo = 0, hi = B;
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (pre[mid] <= gi) lo = mid; else hi = mid;
    }
    return lo;
}

// The appended token ranges whose pages a refreshing scan rebuilds first (the arguments of
// ekv_page_meta_update); nr leading blocks do that, two per (sequence, KV head).
struct RefreshArgs {
    const int32_t *new_start, *new_count;
    int max_new, nr;
};

template <int DT, int D, int G, bool REFRESH>
__device__ __forceinline__ void score_topk_body(const ekv_cache &c, const void *__restrict__ q,
                                                int H_q, float scale, float *__restrict__ scores,
                                                const RefreshArgs &ra)
{
    extern __shared__ int pre[];  // [B + 1], then (refresh) the touched groups [B][2]
    __shared__ int warp_tot[8];
    constexpr int EPC = Chunk<DT>::N;
    constexpr int CPR = 2 * D * Chunk<DT>::kBytes / 16;  // 16-byte chunks per bbox row
    constexpr int W = CPR < 32 ? CPR : 32;                 // lanes per row
    constexpr int LPL = CPR / W;                           // chunks per lane per row
    constexpr int RPI = 32 / W;                            // rows per warp instruction
    constexpr int PG = 8;                                  // pages per work group
    constexpr int NPL = PG / RPI;                          // page slots per lane
    static_assert(NPL <= W, "one result per lane group");

    pdl_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = c.num_kv_heads, B = c.batch, P = c.page_size;
    // Refresh: the groups holding the appended pages of sequence b are tg[2b]..tg[2b + 1]
    // (-1: none). Blocks [0, nr) rebuild those pages' metadata and score their groups (block r:
    // sequence and head r / 2, the first or the last touched group); the other blocks scan the
    // rest and skip them.
    int *tg = pre + B + 1;
    bool fresh = false;
    if constexpr (REFRESH) {
        for (int b = threadIdx.x; b < B; b += blockDim.x) {
            int len, s, n;
            seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
            const bool any = append_range(c, ra.new_start, ra.new_count, ra.max_new, b, len,
                                          false, s, n);
            tg[2 * b] = any ? s / P / PG : -1;
            tg[2 * b + 1] = any ? (s + n - 1) / P / PG : -1;
        }
        fresh = (int)blockIdx.x < ra.nr;
    }
    const long TG = build_group_prefix<PG>(c, pre, warp_tot);
    long lo, hi;
    if constexpr (REFRESH) {
        if (fresh) {
            __shared__ MetaPageShared<D> msm;
            const int bh = blockIdx.x >> 1, b = bh / H, h = bh % H;
            int len, s, n;
            const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
            // a bad range is reported once per sequence, by its head-0 first-group block
            if (!append_range(c, ra.new_start, ra.new_count, ra.max_new, b, len,
                              (blockIdx.x & 1) == 0 && h == 0 && threadIdx.x == 0, s, n))
                return;
            const int g = tg[2 * b + (blockIdx.x & 1)];
            if ((blockIdx.x & 1) && g == tg[2 * b]) return;  // one touched group
            const int p0 = max(s / P, g * PG), p1 = min((s + n - 1) / P, g * PG + PG - 1);
            for (int p = p0; p <= p1; ++p) meta_refresh_page<DT, D>(c, b, h, p, len, msm);
            // the block's metadata stores are visible to its own threads from here on; warp 0
            // scores the group (bbox rows read coherently, not through the read-only path)
            lo = pre[b] + (long)h * ((np + PG - 1) / PG) + g;
            hi = lo + 1;
        } else {
            lo = (long)(blockIdx.x - ra.nr) * TG / (gridDim.x - ra.nr);
            hi = (long)(blockIdx.x - ra.nr + 1) * TG / (gridDim.x - ra.nr);
        }
    } else {
        lo = (long)blockIdx.x * TG / gridDim.x;
        hi = (long)(blockIdx.x + 1) * TG / gridDim.x;
    }
    const char *bbox = static_cast<const char *>(c.meta_bbox);

    // Work group gi -> (sequence, KV head, first page); its page-table entries are fetched
    // one group ahead, so each group's bbox loads wait on one memory latency, not two.
    struct Grp { int bb, hh, j0, np; };
    auto locate = [&](long gi) {
        Grp g;
        g.bb = find_seq(pre, B, gi);
        int len = c.seq_lens[g.bb];
        len = len < 0 ? 0 : (len > c.max_pages * P ? c.max_pages * P : len);
        g.np = (len + P - 1) / P;
        const int ng = (g.np + PG - 1) / PG;
        const int r = (int)(gi - pre[g.bb]);
        g.hh = r / ng;
        g.j0 = (r % ng) * PG;
        return g;
    };
    // block id of page j0 + (lane & 7): -1 past the end, -2 out of range
    auto fetch_blk = [&](const Grp &g) {
        int blk = -1;
        const int jl = g.j0 + (lane & (PG - 1));
        if (jl < g.np) {
            blk = c.page_table[(size_t)g.bb * c.max_pages + jl];
            if (blk < 0 || blk >= c.num_blocks) {
                flag(c.dev_status, EKV_DEV_BAD_BLOCK);
                blk = -2;
            }
        }
        return blk;
    };

    int cur_bh = -1;
    float coef[LPL][EPC];
    long gi = lo + warp;
    Grp nxt = {0, 0, 0, 0};
    int nxt_blk = -1;
    if (gi < hi) {
        nxt = locate(gi);
        nxt_blk = fetch_blk(nxt);
    }
    for (; gi < hi; gi += 8) {
        const Grp cur = nxt;
        const int myblk = nxt_blk;
        const int bh = cur.bb * H + cur.hh;
        if constexpr (REFRESH) {
            const int gg = cur.j0 / PG;  // a group a refresh block scores: not ours
            if (!fresh && gg >= tg[2 * cur.bb] && gg <= tg[2 * cur.bb + 1]) {
                if (gi + 8 < hi) {
                    nxt = locate(gi + 8);
                    nxt_blk = fetch_blk(nxt);
                }
                continue;
            }
        }
        uint4 x[NPL][LPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int blk = __shfl_sync(kFull, myblk, i * RPI + lane / W);
#pragma unroll
            for (int k = 0; k < LPL; ++k) {
                const char *src = bbox + (((size_t)blk * H + cur.hh) * CPR + k * W + lane % W) * 16;
                if (blk < 0)
                    x[i][k] = make_uint4(0, 0, 0, 0);
                else if (REFRESH && fresh)
                    x[i][k] = ld_cg16(src);
                else
                    x[i][k] = ld_stream16(src);
            }
        }
        if (gi + 8 < hi) {
            nxt = locate(gi + 8);
            nxt_blk = fetch_blk(nxt);
        }
        if (bh != cur_bh) {
            cur_bh = bh;
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
                        float qv = load_elem<DT>(q, ((size_t)cur.bb * H_q + cur.hh * G + g) * D + cb + e);
                        a += upper ? fmaxf(qv, 0.f) : fminf(qv, 0.f);
                    }
                    coef[k][e] = a;
                }
            }
        }
        float part[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            part[i] = 0.f;
#pragma unroll
            for (int k = 0; k < LPL; ++k) {
                float f[EPC];
                Chunk<DT>::unpack(x[i][k], f);
#pragma unroll
                for (int e = 0; e < EPC; ++e) part[i] = fmaf(coef[k][e], f[e], part[i]);
            }
        }
        transpose_reduce<NPL, W>(part, lane);
        const int po = transpose_index<NPL, W>(lane, 0) * RPI + lane / W;
        const int blk = __shfl_sync(kFull, myblk, po);
        if (((lane % W) % (W / NPL)) == 0 && cur.j0 + po < cur.np)
            scores[(size_t)bh * c.max_pages + cur.j0 + po] = blk >= 0 ? scale * part[0] : -INFINITY;
    }
}

template <int DT, int D, int G>
__global__ void __launch_bounds__(256)
score_topk_kernel(ekv_cache c, const void *__restrict__ q, int H_q, float scale,
                  float *__restrict__ scores)
{
    score_topk_body<DT, D, G, false>(c, q, H_q, scale, scores, RefreshArgs{});
}

// ekv_page_meta_update of a short append followed by the top-k scan, in one launch: blocks
// [0, ra.nr) rebuild the appended pages' metadata (meta_refresh_page, as the short-append
// kernel does) and score the 8-page groups holding them; the other blocks scan every other
// group. The results are those of the two calls, bit for bit; the refresh runs under the scan
// instead of before it.
template <int DT, int D, int G>
__global__ void __launch_bounds__(256, DT == EKV_BF16 ? 4 : 1)
score_refresh_topk_kernel(ekv_cache c, const void *__restrict__ q, int H_q, float scale,
                          float *__restrict__ scores, RefreshArgs ra)
{
    score_topk_body<DT, D, G, true>(c, q, H_q, scale, scores, ra);
}

template <int DT, int D, int G>
__global__ void __launch_bounds__(256)
score_gauss_kernel(ekv_cache c, const void *__restrict__ q, int H_q, float scale,
                   float *__restrict__ scores)
{
    // Lane l owns coordinates [l * VEC, (l + 1) * VEC) of all four metadata rows of a page
    // (kmin, kmax, mean, variance), so the query coefficients it needs are just q_g there.
    extern __shared__ int pre[];
    __shared__ int warp_tot[8];
    constexpr int VEC = D / 32;
    constexpr int PGG = G >= 8 ? 1 : 8 / G;  // pages per work group
    constexpr int NV = PGG * G;              // 8 values per output kind per lane

    pdl_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = c.num_kv_heads, B = c.batch, P = c.page_size;
    const long TG = build_group_prefix<PGG>(c, pre, warp_tot);
    const long lo = (long)blockIdx.x * TG / gridDim.x;
    const long hi = (long)(blockIdx.x + 1) * TG / gridDim.x;

    // Work group gi -> (sequence, KV head, first page); as in the top-k scan, a group's
    // page-table entries are fetched one group ahead, so its metadata loads wait on one memory
    // latency, not two.
    struct Grp { int bb, hh, j0, np; };
    auto locate = [&](long gi) {
        Grp g;
        g.bb = find_seq(pre, B, gi);
        int len = c.seq_lens[g.bb];
        len = len < 0 ? 0 : (len > c.max_pages * P ? c.max_pages * P : len);
        g.np = (len + P - 1) / P;
        const int ng = (g.np + PGG - 1) / PGG;
        const int r = (int)(gi - pre[g.bb]);
        g.hh = r / ng;
        g.j0 = (r % ng) * PGG;
        return g;
    };
    auto fetch_blk = [&](const Grp &g) {  // block of page j0 + lane % PGG: -1 past the end, -2 bad
        int blk = -1;
        const int jl = g.j0 + lane % PGG;
        if (jl < g.np) {
            blk = c.page_table[(size_t)g.bb * c.max_pages + jl];
            if (blk < 0 || blk >= c.num_blocks) {
                flag(c.dev_status, EKV_DEV_BAD_BLOCK);
                blk = -2;
            }
        }
        return blk;
    };

    int cur_bh = -1;
    float qv[G][VEC];
    long gi = lo + warp;
    Grp nxt = {0, 0, 0, 0};
    int nxt_blk = -1;
    if (gi < hi) {
        nxt = locate(gi);
        nxt_blk = fetch_blk(nxt);
    }
    for (; gi < hi; gi += 8) {
        const Grp cur = nxt;
        const int myblk = nxt_blk;
        const int bb = cur.bb, hh = cur.hh, j0 = cur.j0, np = cur.np;
        const int bh = bb * H + hh;
        if (bh != cur_bh) {
            cur_bh = bh;
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < VEC; ++e)
                    qv[g][e] = load_elem<DT>(q, ((size_t)bb * H_q + hh * G + g) * D + lane * VEC + e);
        }
        float kn[PGG][VEC], kx[PGG][VEC], mu[PGG][VEC], vr[PGG][VEC];
#pragma unroll
        for (int i = 0; i < PGG; ++i) {
            const int blk = __shfl_sync(kFull, myblk, i);
            const size_t base = ((size_t)(blk < 0 ? 0 : blk) * H + hh) * 2 * D + lane * VEC;
            if (blk >= 0) {
                load_vec_nc<DT, VEC>(static_cast<const char *>(c.meta_bbox) + base * Chunk<DT>::kBytes, kn[i]);
                load_vec_nc<DT, VEC>(static_cast<const char *>(c.meta_bbox) + (base + D) * Chunk<DT>::kBytes, kx[i]);
                load_vec_nc<EKV_F32, VEC>(c.meta_mom + base, mu[i]);
                load_vec_nc<EKV_F32, VEC>(c.meta_mom + base + D, vr[i]);
            } else {
#pragma unroll
                for (int e = 0; e < VEC; ++e) { kn[i][e] = 0.f; kx[i][e] = 0.f; mu[i][e] = 0.f; vr[i][e] = 0.f; }
            }
        }
        if (gi + 8 < hi) {
            nxt = locate(gi + 8);
            nxt_blk = fetch_blk(nxt);
        }
        float pu[NV], pm[NV], pv[NV];
#pragma unroll
        for (int i = 0; i < PGG; ++i)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float u = 0.f, m = 0.f, v = 0.f;
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float qe = qv[g][e];
                    u += fmaxf(qe * kn[i][e], qe * kx[i][e]);
                    m = fmaf(qe, mu[i][e], m);
                    v = fmaf(qe * qe, vr[i][e], v);
                }
                pu[i * G + g] = u; pm[i * G + g] = m; pv[i * G + g] = v;
            }
        transpose_reduce<NV, 32>(pu, lane);
        transpose_reduce<NV, 32>(pm, lane);
        transpose_reduce<NV, 32>(pv, lane);
        const int idx = transpose_index<NV, 32>(lane, 0);
        const int i = idx / G, g = idx % G;
        const int blk = __shfl_sync(kFull, myblk, i);
        if ((lane & (32 / NV - 1)) == 0 && j0 + i < np) {
            float *out = scores + ((size_t)bb * H_q + hh * G + g) * 3 * c.max_pages + j0 + i;
            const bool ok = blk >= 0;
            out[0] = ok ? scale * pu[0] : -INFINITY;
            out[c.max_pages] = ok ? scale * pm[0] : 0.f;
            out[2 * (size_t)c.max_pages] = ok ? scale * scale * pv[0] : 0.f;
        }
    }
}

template <int DT, int D, int G>
static cudaError_t launch_score_t(const ekv_cache &c, const void *q, int H_q, float scale,
                                  int policy, float *scores, cudaStream_t st, bool pdl)
{
    const size_t smem = sizeof(int) * (c.batch + 1);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (policy == EKV_SEL_TOPK) {
        auto k = score_topk_kernel<DT, D, G>;
        cfg.gridDim = dim3(persistent_grid_size((const void *)k, 256, smem));
        return cudaLaunchKernelEx(&cfg, k, c, q, H_q, scale, scores);
    }
    auto k = score_gauss_kernel<DT, D, G>;
    cfg.gridDim = dim3(persistent_grid_size((const void *)k, 256, smem));
    return cudaLaunchKernelEx(&cfg, k, c, q, H_q, scale, scores);
}

template <int DT, int D>
static cudaError_t launch_score_g(const ekv_cache &c, const void *q, int H_q, float scale,
                                  int policy, float *scores, cudaStream_t st, bool pdl)
{
    switch (H_q / c.num_kv_heads) {
    case 1: return launch_score_t<DT, D, 1>(c, q, H_q, scale, policy, scores, st, pdl);
    case 2: return launch_score_t<DT, D, 2>(c, q, H_q, scale, policy, scores, st, pdl);
    case 4: return launch_score_t<DT, D, 4>(c, q, H_q, scale, policy, scores, st, pdl);
    default: return launch_score_t<DT, D, 8>(c, q, H_q, scale, policy, scores, st, pdl);
    }
}

cudaError_t launch_score_pages(const ekv_cache &c, const void *q, int H_q, float scale,
                               int policy, float *scores, cudaStream_t st, bool pdl)
{
    if (c.dtype == EKV_BF16)
        return c.head_dim == 128 ? launch_score_g<EKV_BF16, 128>(c, q, H_q, scale, policy, scores, st, pdl)
                                 : launch_score_g<EKV_BF16, 64>(c, q, H_q, scale, policy, scores, st, pdl);
    return c.head_dim == 128 ? launch_score_g<EKV_F32, 128>(c, q, H_q, scale, policy, scores, st, pdl)
                             : launch_score_g<EKV_F32, 64>(c, q, H_q, scale, policy, scores, st, pdl);
}


template <int DT, int D, int G>
static cudaError_t launch_refresh_t(const ekv_cache &c, const void *q, int H_q, float scale,
                                    float *scores, RefreshArgs ra, cudaStream_t st, bool pdl,
                                    bool *launched)
{
    auto k = score_refresh_topk_kernel<DT, D, G>;
    const size_t smem = sizeof(int) * (3 * (size_t)c.batch + 1);
    const int grid = persistent_grid_size((const void *)k, 256, smem);
    // The refresh blocks come out of the scan's single wave: only when they are few (at most a
    // sixteenth of the grid) is the scan they slow down cheaper than a launch of its own.
    ra.nr = 2 * c.batch * c.num_kv_heads;
    *launched = (long long)ra.nr * 16 <= grid;
    if (!*launched) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cfg.gridDim = dim3(grid);
    return cudaLaunchKernelEx(&cfg, k, c, q, H_q, scale, scores, ra);
}

template <int DT, int D>
static cudaError_t launch_refresh_g(const ekv_cache &c, const void *q, int H_q, float scale,
                                    float *scores, RefreshArgs ra, cudaStream_t st, bool pdl,
                                    bool *launched)
{
    switch (H_q / c.num_kv_heads) {
    case 1: return launch_refresh_t<DT, D, 1>(c, q, H_q, scale, scores, ra, st, pdl, launched);
    case 2: return launch_refresh_t<DT, D, 2>(c, q, H_q, scale, scores, ra, st, pdl, launched);
    case 4: return launch_refresh_t<DT, D, 4>(c, q, H_q, scale, scores, ra, st, pdl, launched);
    default: return launch_refresh_t<DT, D, 8>(c, q, H_q, scale, scores, ra, st, pdl, launched);
    }
}

cudaError_t launch_page_meta_update(const ekv_cache &c, const int32_t *new_start,
                                    const int32_t *new_count, int max_new, cudaStream_t st);

// ekv_page_meta_update then ekv_score_pages. A short append (at most 2 P tokens per sequence)
// under the top-k policy with few (sequence, KV head) pairs runs as one refreshing scan;
// otherwise the two kernels run one after the other.
cudaError_t launch_refresh_score_pages(const ekv_cache &c, const int32_t *new_start,
                                       const int32_t *new_count, int max_new, const void *q,
                                       int H_q, float scale, int policy, float *scores,
                                       cudaStream_t st, bool pdl)
{
    if (max_new == 0) return launch_score_pages(c, q, H_q, scale, policy, scores, st, pdl);
    if (policy == EKV_SEL_TOPK && max_new <= 2 * c.page_size) {
        const RefreshArgs ra = {new_start, new_count, max_new, 0};
        bool launched = false;
        cudaError_t e;
        if (c.dtype == EKV_BF16)
            e = c.head_dim == 128 ? launch_refresh_g<EKV_BF16, 128>(c, q, H_q, scale, scores, ra, st, pdl, &launched)
                                  : launch_refresh_g<EKV_BF16, 64>(c, q, H_q, scale, scores, ra, st, pdl, &launched);
        else
            e = c.head_dim == 128 ? launch_refresh_g<EKV_F32, 128>(c, q, H_q, scale, scores, ra, st, pdl, &launched)
                                  : launch_refresh_g<EKV_F32, 64>(c, q, H_q, scale, scores, ra, st, pdl, &launched);
        if (e != cudaSuccess || launched) return e;
    }
    cudaError_t e = launch_page_meta_update(c, new_start, new_count, max_new, st);
    if (e != cudaSuccess) return e;
    return launch_score_pages(c, q, H_q, scale, policy, scores, st, pdl);
}

}  // namespace ekv
