// select.cu -- candidate page selection (EntmaxKV technical summary, §2.B).
//
// Top-k (§2.B.1), one 1024-thread CTA per (sequence, KV head): an exact radix select over
// order-preserving 32-bit keys of the fp32 scores (11 + 11 + 10 bits; histograms with
// warp-aggregated shared-memory increments, so a run of nearly equal scores does not serialise
// on one counter) finds the k-th largest key T and how many keys equal to T are taken; a
// block scan then emits the kept pages in ascending order, equal scores going to the lower
// page index.
//
// Gaussian-aware (§2.B.2), one CTA per (sequence, KV head), one warp per query of the group:
// tau-hat solves F(tau) = sum_j n_j E[(X_j - tau)_+^(1/(alpha-1))] = 1 with
// X_j ~ N((alpha-1) m_j, (alpha-1)^2 v_j). F is convex and decreasing, so Newton's method
// started at max_j a_j - 1 (where F >= 1 by Jensen) climbs monotonically to the root. Pages
// with a_j + 8 b_j <= max_j a_j - 1 contribute less than 1e-16 n_j b_j^2 to F at every tau on
// that path and are dropped before the iterations; the rest are kept in shared memory. Then a
// block scan keeps page j iff some query g has (alpha-1) UB_gj > tau_hat_g - Delta.
#include "cluster.cuh"
#include "topk_cta.cuh"

namespace ekv {

__device__ __forceinline__ uint32_t order_key(float x)
{
    if (x != x) return 0u;                  // NaN sorts below everything
    uint32_t u = __float_as_uint(x + 0.0f);  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelThreads = 1024;
constexpr int kSmemKeys = 16384;  // keys staged in shared memory (larger n reads them from L2)
constexpr int kBoundaryMax = 256; // boundary-bin entries resolved by rank counting

// The bin holding the k-th largest key: counts in descending bin order (thread t owns bins
// nb-1-BPT*t ... nb-BPT-BPT*t), a block scan, and the one thread whose bins cross k writes the
// bin and the count of keys in the bins above it. Ends with a barrier.
template <int NT, int BPT>
__device__ __forceinline__ void find_bin_from_top(const int *hist, int nb, int k, int *warp_tot,
                                                  int *s_bin, int *s_above)
{
    const int tid = threadIdx.x;
    int cnt[BPT], sum = 0;
#pragma unroll
    for (int r = 0; r < BPT; ++r) {
        const int bin = nb - 1 - BPT * tid - r;
        cnt[r] = bin >= 0 ? hist[bin] : 0;
        sum += cnt[r];
    }
    const int incl = block_incl_scan<NT>(sum, warp_tot, nullptr);
    int run = incl - sum;
#pragma unroll
    for (int r = 0; r < BPT; ++r) {
        if (cnt[r] > 0 && run < k && k <= run + cnt[r]) {
            *s_bin = nb - 1 - BPT * tid - r;
            *s_above = run;
        }
        run += cnt[r];
    }
    __syncthreads();
}

// Exact radix select on the order-preserving keys (11 + 11 + 10 bits) and emission of the
// kept pages in ascending order. `key(j)` returns the key of page j.
template <class KeyFn>
__device__ void radix_select_emit(int n, int kk, KeyFn key, int *hist, int *warp_tot, int *s_bin,
                                  int *s_above, int32_t *out)
{
    constexpr int NT = kSelThreads;
    const int tid = threadIdx.x, lane = tid & 31;
    uint32_t prefix = 0, mask = 0;
    int remaining = kk;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int i = tid; i < 2048; i += NT) hist[i] = 0;
        __syncthreads();
        for (int j0 = 0; j0 < n; j0 += NT) {
            const int j = j0 + tid;
            int bin = -1;
            if (j < n) {
                const uint32_t u = key(j);
                if ((u & mask) == prefix) bin = (int)((u >> shift) & (uint32_t)(nb - 1));
            }
            const unsigned peers = __match_any_sync(kFull, bin);
            if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
        }
        __syncthreads();
        find_bin_from_top<NT, 2048 / NT>(hist, nb, remaining, warp_tot, s_bin, s_above);
        remaining -= *s_above;
        prefix |= (uint32_t)*s_bin << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        const bool whole_bin = remaining == hist[*s_bin];
        __syncthreads();
        if (whole_bin) break;  // every key matching the prefix is kept: lower bits cannot matter
    }
    const uint32_t T = prefix;
    auto cmp = [&](uint32_t u) -> int { const uint32_t um = u & mask; return um > T ? 1 : (um == T ? 0 : -1); };
    // emission in page order: warp w owns a contiguous page range; ties at T are kept while
    // their rank among all ties (in page order) is below `remaining`
    const int warp = tid >> 5;
    const int per = (n + NT / 32 - 1) / (NT / 32);
    const int j0 = warp * per, j1 = j0 + per < n ? j0 + per : n;
    int n_above = 0, n_tie = 0;
    for (int j = j0 + lane; j - lane < j1; j += 32) {
        const int c = j < j1 ? cmp(key(j)) : -1;
        n_above += __popc(__ballot_sync(kFull, c > 0));
        n_tie += __popc(__ballot_sync(kFull, c == 0));
    }
    if (lane == 0) { hist[warp] = n_above; hist[32 + warp] = n_tie; }
    __syncthreads();
    if (warp == 0) {
        const int a = hist[lane], t = hist[32 + lane];
        const int ia = warp_incl_scan(a), it = warp_incl_scan(t);
        hist[64 + lane] = ia - a;   // kept-above before this warp
        hist[96 + lane] = it - t;   // ties before this warp
    }
    __syncthreads();
    int tie_rank = hist[96 + warp];
    int pos = hist[64 + warp] + (tie_rank < remaining ? tie_rank : remaining);
    for (int j = j0 + lane; j - lane < j1; j += 32) {
        const int c = j < j1 ? cmp(key(j)) : -1;
        const unsigned tb = __ballot_sync(kFull, c == 0);
        const bool keep = c > 0 || (c == 0 && tie_rank + __popc(tb & ((1u << lane) - 1u)) < remaining);
        const unsigned kb = __ballot_sync(kFull, keep);
        if (keep) out[pos + __popc(kb & ((1u << lane) - 1u))] = j;
        pos += __popc(kb);
        tie_rank += __popc(tb);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads)
select_topk_kernel(const float *__restrict__ scores, int H, int max_pages, int P,
                   const int32_t *__restrict__ seq_lens, int k, int32_t *__restrict__ sel_idx,
                   int32_t *__restrict__ sel_count, int max_sel, uint32_t *status)
{
    // The keys of one (sequence, KV head) go to shared memory once (all loads in flight
    // together). One histogram pass over 2048 bins that split the [min, max] key range evenly
    // finds the bin holding the k-th largest key; the few keys of that bin are ranked exactly
    // by (key descending, page ascending). Heavy ties (a large boundary bin) or more than
    // kSmemKeys pages take the three-pass radix select instead.
    constexpr int NT = kSelThreads;
    constexpr int NB = 2048;
    extern __shared__ uint32_t keys[];  // [min(n, kSmemKeys)]
    __shared__ int hist[2048];
    __shared__ int warp_tot[32];
    __shared__ int s_bin, s_above, s_cnt;
    __shared__ uint32_t s_umin, s_umax;
    __shared__ uint32_t bu[kBoundaryMax];
    __shared__ int bj[kBoundaryMax];
    __shared__ uint32_t kept_bits[kSmemKeys / 32];
    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.x, b = blockIdx.y;
    const int bh = b * H + h;
    const int n = seq_pages(seq_lens, b, P, max_pages, h == 0 ? status : nullptr, nullptr);
    const float *S = scores + (size_t)bh * max_pages;
    int32_t *out = sel_idx + (size_t)bh * max_sel;
    const int kk = k < n ? k : n;

    if (kk == n) {  // every page is kept
        for (int j = tid; j < max_sel; j += NT) out[j] = j < n ? j : -1;
        if (tid == 0) sel_count[bh] = n;
        pdl_trigger();
        return;
    }
    if (n > kSmemKeys) {
        radix_select_emit(n, kk, [&](int j) { return order_key(__ldcg(S + j)); }, hist, warp_tot,
                          &s_bin, &s_above, out);
        for (int j = kk + tid; j < max_sel; j += NT) out[j] = -1;
        if (tid == 0) sel_count[bh] = kk;
        pdl_trigger();
        return;
    }

    uint32_t umin = 0xffffffffu, umax = 0;
    if ((max_pages & 3) == 0) {
        const float4 *S4 = reinterpret_cast<const float4 *>(S);
        const int n4 = n >> 2;
#pragma unroll 4
        for (int i = tid; i < n4; i += NT) {
            const float4 v = __ldcg(S4 + i);
            const uint32_t u0 = order_key(v.x), u1 = order_key(v.y), u2 = order_key(v.z), u3 = order_key(v.w);
            keys[4 * i] = u0; keys[4 * i + 1] = u1; keys[4 * i + 2] = u2; keys[4 * i + 3] = u3;
            umin = min(min(umin, u0), min(u1, min(u2, u3)));
            umax = max(max(umax, u0), max(u1, max(u2, u3)));
        }
        for (int j = 4 * n4 + tid; j < n; j += NT) {
            const uint32_t u = order_key(__ldcg(S + j));
            keys[j] = u;
            umin = min(umin, u);
            umax = max(umax, u);
        }
    } else {
#pragma unroll 4
        for (int j = tid; j < n; j += NT) {
            const uint32_t u = order_key(__ldcg(S + j));
            keys[j] = u;
            umin = min(umin, u);
            umax = max(umax, u);
        }
    }
    for (int i = tid; i < NB; i += NT) hist[i] = 0;
    for (int i = tid; i < kSmemKeys / 32; i += NT) kept_bits[i] = 0;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        umin = min(umin, __shfl_xor_sync(kFull, umin, o));
        umax = max(umax, __shfl_xor_sync(kFull, umax, o));
    }
    if (tid == 0) { s_umin = 0xffffffffu; s_umax = 0; s_cnt = 0; }
    __syncthreads();
    if (lane == 0) { atomicMin(&s_umin, umin); atomicMax(&s_umax, umax); }
    __syncthreads();
    umin = s_umin;
    umax = s_umax;
    // monotone bin of a key: floor((u - umin) * NB / (umax - umin + 1)) in fp32 (rounding is
    // monotone, so equal keys share a bin and bin order never contradicts key order)
    const float bscale = (float)NB / ((float)(umax - umin) + 1.0f);
    auto bin_of = [&](uint32_t u) {
        const int bb = (int)((float)(u - umin) * bscale);
        return bb < NB - 1 ? bb : NB - 1;
    };

    for (int j = tid; j < n; j += NT) atomicAdd(&hist[bin_of(keys[j])], 1);
    __syncthreads();
    // counts in descending bin order: thread t owns bins NB-1-2t and NB-2-2t
    find_bin_from_top<NT, NB / NT>(hist, NB, kk, warp_tot, &s_bin, &s_above);
    const int B = s_bin, r = kk - s_above, cB = hist[B];

    if (cB > kBoundaryMax) {  // heavy ties around the k-th key
        radix_select_emit(n, kk, [&](int j) { return keys[j]; }, hist, warp_tot, &s_bin,
                          &s_above, out);
    } else {
        for (int j = tid; j < n; j += NT)
            if (bin_of(keys[j]) == B) {
                const int pos = atomicAdd(&s_cnt, 1);
                bu[pos] = keys[j];
                bj[pos] = j;
            }
        __syncthreads();
        if (tid < cB) {
            const uint32_t u = bu[tid];
            const int j = bj[tid];
            int rank = 0;
            for (int m = 0; m < cB; ++m) rank += bu[m] > u || (bu[m] == u && bj[m] < j);
            if (rank < r) atomicOr(&kept_bits[j >> 5], 1u << (j & 31));
        }
        __syncthreads();
        // emission in page order: warp w owns a contiguous page range
        const int per = (n + NT / 32 - 1) / (NT / 32);
        const int j0 = warp * per, j1 = j0 + per < n ? j0 + per : n;
        auto kept = [&](int j) {
            const int bb = bin_of(keys[j]);
            return bb > B || (bb == B && (kept_bits[j >> 5] >> (j & 31) & 1u));
        };
        int mine = 0;
        for (int j = j0 + lane; j - lane < j1; j += 32)
            mine += __popc(__ballot_sync(kFull, j < j1 && kept(j)));
        if (lane == 0) warp_tot[warp] = mine;
        __syncthreads();
        if (warp == 0) {
            const int v = warp_tot[lane];
            warp_tot[lane] = warp_incl_scan(v) - v;
        }
        __syncthreads();
        int pos = warp_tot[warp];
        for (int j = j0 + lane; j - lane < j1; j += 32) {
            const bool keep = j < j1 && kept(j);
            const unsigned kb = __ballot_sync(kFull, keep);
            if (keep) out[pos + __popc(kb & ((1u << lane) - 1u))] = j;
            pos += __popc(kb);
        }
    }
    for (int j = kk + tid; j < max_sel; j += NT) out[j] = -1;
    if (tid == 0) sel_count[bh] = kk;
    pdl_trigger();
}

// The same selection with each thread's keys in registers, for n <= R * kSelThreads pages:
// thread t owns pages [t R, t R + R), loaded as float4 where the rows allow it (coalesced),
// and cta_topk finds the kept set; one block scan of the threads' kept counts places every
// thread's kept pages, in ascending order.
template <int R>
__global__ void __launch_bounds__(kSelThreads)
select_topk_reg_kernel(const float *__restrict__ scores, int H, int max_pages, int P,
                       const int32_t *__restrict__ seq_lens, int k, int32_t *__restrict__ sel_idx,
                       int32_t *__restrict__ sel_count, int max_sel, uint32_t *status)
{
    constexpr int NT = kSelThreads;
    __shared__ TopkShared sh;
    pdl_wait();
    const int tid = threadIdx.x;
    const int h = blockIdx.x, b = blockIdx.y;
    const int bh = b * H + h;
    const float *S = scores + (size_t)bh * max_pages;
    // every float4 of the row issued at once, before the sequence length is known (entries
    // past the last page are ignored)
    const int j0 = tid * R;
    uint32_t u[R];
    if ((max_pages & 3) == 0) {
        const float4 *S4 = reinterpret_cast<const float4 *>(S + j0);
#pragma unroll
        for (int q4 = 0; q4 < R / 4; ++q4) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j0 + 4 * q4 < max_pages) v = __ldcg(S4 + q4);  // max_pages % 4 == 0: inside the row
            u[4 * q4] = topk_order_key(v.x);
            u[4 * q4 + 1] = topk_order_key(v.y);
            u[4 * q4 + 2] = topk_order_key(v.z);
            u[4 * q4 + 3] = topk_order_key(v.w);
        }
    } else {
#pragma unroll
        for (int r = 0; r < R; ++r) u[r] = j0 + r < max_pages ? topk_order_key(__ldcg(S + j0 + r)) : 0u;
    }
    const int n = seq_pages(seq_lens, b, P, max_pages, h == 0 ? status : nullptr, nullptr);
    int32_t *out = sel_idx + (size_t)bh * max_sel;
    const int kk = k < n ? k : n;
    if (kk == n) {  // every page is kept
        for (int j = tid; j < max_sel; j += NT) out[j] = j < n ? j : -1;
        if (tid == 0) sel_count[bh] = n;
        return;
    }
    bool keep[R];
    const int mine = cta_topk<NT, R>(u, n, kk, sh, keep);
    int pos = block_incl_scan<NT>(mine, sh.warp_tot, nullptr) - mine;
#pragma unroll
    for (int r = 0; r < R; ++r)
        if (keep[r] && pos < kk) out[pos++] = j0 + r;
    for (int j = kk + tid; j < max_sel; j += NT) out[j] = -1;
    if (tid == 0) sel_count[bh] = kk;
}

// ---------------------------------------------------------------------------- Gaussian-aware
// E[(X - tau)_+^p] for X ~ N(a, b^2), p = 1 (alpha = 2) or 2 (alpha = 1.5), and its
// derivative in tau, in fp32. Phi(u) = erfc(-u / sqrt 2) / 2, phi(u) = exp(-u^2 / 2) / sqrt(2 pi).
__device__ __forceinline__ void trunc_moment(float a, float b, float tau, bool sparsemax,
                                             float &E, float &dE)
{
    const float r = a - tau;
    if (b <= 0.f) {
        const float rp = r > 0.f ? r : 0.f;
        E = sparsemax ? rp : rp * rp;
        dE = sparsemax ? (r > 0.f ? -1.f : 0.f) : -2.f * rp;
        return;
    }
    const float u = r / b;
    const float Phi = 0.5f * erfcf(-u * 0.70710678118654752f);
    const float phi = 0.39894228040143268f * __expf(-0.5f * u * u);
    if (sparsemax) {
        E = r * Phi + b * phi;
        dE = -Phi;
    } else {
        E = (r * r + b * b) * Phi + r * b * phi;
        dE = -2.f * (r * Phi + b * phi);
    }
}

// Newton step for F^(1/p) = 1 given F and F' (p = 1 sparsemax, p = 2 1.5-entmax):
// (F^(1/p) - 1) / -(F^(1/p))'.
__device__ __forceinline__ double newton_step(double F, double dF, bool sparsemax)
{
    if (sparsemax) return (F - 1.0) / -dF;
    const double r = sqrt(F);
    return (r - 1.0) * 2.0 * r / -dF;
}

// The same moments in fp64, for the final Newton steps.
__device__ __forceinline__ void trunc_moment_d(double a, double b, double tau, bool sparsemax,
                                               double &E, double &dE)
{
    const double r = a - tau;
    if (b <= 0.0) {
        const double rp = r > 0.0 ? r : 0.0;
        E = sparsemax ? rp : rp * rp;
        dE = sparsemax ? (r > 0.0 ? -1.0 : 0.0) : -2.0 * rp;
        return;
    }
    const double u = r / b;
    const double Phi = 0.5 * erfc(-u * 0.70710678118654752440);
    const double phi = 0.39894228040143267794 * exp(-0.5 * u * u);
    if (sparsemax) {
        E = r * Phi + b * phi;
        dE = -Phi;
    } else {
        E = (r * r + b * b) * Phi + r * b * phi;
        dE = -2.0 * (r * Phi + b * phi);
    }
}

constexpr int kGaussSmemBytes = 200 * 1024;  // dynamic shared memory of one CTA at most
constexpr int kGaussList = 64;                // survivors gathered for warp 0 to iterate on alone

// One CTA of 4 warps per query; the G CTAs of a (sequence, KV head) form a thread-block
// cluster. Each warp owns a slice of the pages and a slice of the survivor list in shared
// memory: (a_j, b_j, n_j) with a = (alpha-1) m, b = (alpha-1) sqrt(v) and n_j the page's token
// count. When the slice fits, the warp stages its pages' model with all loads in flight;
// otherwise it reads them from global memory for the maximum and keeps only the pages that
// survive the first prune (more than the capacity and it walks global memory on every
// iteration).
//
// tau solves F(tau) = sum_j n_j E[(X_j - tau)_+^p] = 1. F^(1/p) is convex and decreasing (an
// L^p norm of (X - tau)_+, each term convex in tau) and close to linear well left of the root,
// so Newton on F^(1/p) = 1 from tau0 = max_j a_j - 1 (where F >= 1) rises monotonically onto
// the root in a few steps. Pages with a + 8 b <= tau contribute below 1e-14 of their count.
// When the first prune at tau0 leaves at most kGaussList pages they are gathered into one list
// that warp 0 iterates on alone (no barrier per step); larger lists keep every warp on its
// slice, with the sums combined each step. Survivors are pruned again every fourth step. The fp32 iterates stop
// within about 1e-5 of the root; a few Newton steps with fp64 moments finish it.
//
// Each CTA then stores its tau-hat into every CTA of the cluster; after a cluster barrier CTA
// g takes the g-th slice of the pages and marks every page with (alpha-1) UB_j > tau_g - delta
// for some query g of the group (or the Gaussian estimate of the page maximum, est_max), the
// slices' counts are exchanged the same way, and each CTA writes its kept pages at its offset,
// in ascending page order.
template <int G>
__global__ void __launch_bounds__(128)
select_gauss_kernel(const float *__restrict__ scores, int H, int max_pages, int P,
                    const int32_t *__restrict__ seq_lens, float alpha, float delta,
                    int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_count, int max_sel,
                    float *__restrict__ tau_hat, uint32_t *status, int capw, bool est_max)
{
    constexpr int NT = 128, NW = 4;
    extern __shared__ float gdyn[];  // [NW][3][capw] survivor slices | [3][kGaussList] list | keep bits
    __shared__ double s_part[2][NW][2];
    __shared__ float s_amax[NW];
    __shared__ int s_cnt[NW];
    __shared__ double s_tau[G];  // every query's tau-hat (stored by the cluster)
    __shared__ int s_kept[G];    // kept pages of every CTA's slice (stored by the cluster)
    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = blockIdx.x % G, h = blockIdx.x / G, b = blockIdx.y, bh = b * H + h;
    const int H_q = H * G, hq = h * G + g;
    int len;
    const int n = seq_pages(seq_lens, b, P, max_pages, h == 0 && g == 0 ? status : nullptr, &len);
    const bool sparsemax = alpha == 2.0f;
    const float am1 = alpha - 1.0f;
    float *la = gdyn + (size_t)NW * 3 * capw, *lb = la + kGaussList, *ln = lb + kGaussList;
    unsigned *bits = reinterpret_cast<unsigned *>(ln + kGaussList);

    {
        const float *sc = scores + ((size_t)b * H_q + hq) * 3 * max_pages;
        const float *m = sc + max_pages, *v = sc + 2 * (size_t)max_pages;
        float *sa = gdyn + (size_t)warp * 3 * capw, *sb = sa + capw, *sn = sb + capw;
        const int per = (n + NW - 1) / NW;
        const int p0 = min(warp * per, n), p1 = min(p0 + per, n);
        const bool staged = p1 - p0 <= capw;
        auto page_n = [&](int j) { return (float)(len - j * P < P ? len - j * P : P); };
        auto model = [&](int j, float &aj, float &bj) {
            aj = am1 * __ldcg(m + j);
            bj = am1 * sqrtf(fmaxf(__ldcg(v + j), 0.f));
        };
        float amax = -INFINITY;
        if (staged) {
            for (int j0 = p0; j0 < p1; j0 += 512) {  // 16 loads of (m, v) per lane in flight
                float av[16], bv[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int j = j0 + u * 32 + lane;
                    av[u] = -INFINITY; bv[u] = 0.f;
                    if (j < p1) model(j, av[u], bv[u]);
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int j = j0 + u * 32 + lane;
                    if (j < p1) {
                        sa[j - p0] = av[u]; sb[j - p0] = bv[u]; sn[j - p0] = page_n(j);
                        amax = fmaxf(amax, av[u]);
                    }
                }
            }
        } else {
            for (int j0 = p0; j0 < p1; j0 += 256) {
                float mv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int j = j0 + u * 32 + lane;
                    mv[u] = j < p1 ? __ldcg(m + j) : -INFINITY;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) amax = fmaxf(amax, am1 * mv[u]);
            }
        }
        amax = warp_max(amax);
        if (lane == 0) s_amax[warp] = amax;
        __syncthreads();
        amax = s_amax[0];
#pragma unroll
        for (int k = 1; k < NW; ++k) amax = fmaxf(amax, s_amax[k]);
        const double tau0 = (double)amax - 1.0;

        // first prune: pages that can still contribute at tau >= amax - 1
        int cnt = 0;
        for (int j0 = p0; j0 < p1; j0 += 32) {
            const int j = j0 + lane;
            float aj = 0.f, bj = 0.f, nj = 0.f;
            bool keep = false;
            if (j < p1) {
                if (staged) { aj = sa[j - p0]; bj = sb[j - p0]; nj = sn[j - p0]; }
                else { model(j, aj, bj); nj = page_n(j); }
                keep = (double)aj + 8.0 * (double)bj > tau0;
            }
            const unsigned bal = __ballot_sync(kFull, keep);
            const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
            __syncwarp();
            if (keep && pos < capw) { sa[pos] = aj; sb[pos] = bj; sn[pos] = nj; }
            cnt += __popc(bal);
            __syncwarp();
        }
        if (lane == 0) s_cnt[warp] = cnt;
        __syncthreads();
        int total = 0, before = 0;
        bool any_over = false;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            total += s_cnt[w];
            before += w < warp ? s_cnt[w] : 0;
            any_over = any_over || s_cnt[w] > capw;
        }
        const bool solo = !any_over && total <= kGaussList;  // the same in every thread
        if (solo) {  // gather the survivors into one list
            for (int i = lane; i < cnt; i += 32) {
                la[before + i] = sa[i];
                lb[before + i] = sb[i];
                ln[before + i] = sn[i];
            }
            __syncthreads();
        }

        // Newton on the list (a, b, n)[0, cnt), or on the warp's pages in global memory (glob);
        // `reduce` adds the warps' totals of F, F' over the participating warps.
        auto newton = [&](float *xa, float *xb, float *xn, int cnt, bool glob, auto &&reduce) {
            double tau = tau0;
            if (n == 0) return -(double)INFINITY;
            bool settled = false;  // the fp32 iterates met their step tolerance
#pragma unroll 1
            for (int it = 0; it < 48; ++it) {
                float F = 0.f, dF = 0.f;
                const float tf = (float)tau;
                if (!glob) {
#pragma unroll 2
                    for (int i = lane; i < cnt; i += 32) {
                        float E, dE;
                        trunc_moment(xa[i], xb[i], tf, sparsemax, E, dE);
                        F = fmaf(xn[i], E, F);
                        dF = fmaf(xn[i], dE, dF);
                    }
                } else {
                    for (int j = p0 + lane; j < p1; j += 32) {
                        float aj, bj, E, dE;
                        model(j, aj, bj);
                        trunc_moment(aj, bj, tf, sparsemax, E, dE);
                        F = fmaf(page_n(j), E, F);
                        dF = fmaf(page_n(j), dE, dF);
                    }
                }
                double Fs, dFs;  // fp32 warp sums are enough for these iterates
                reduce((double)warp_sum(F), (double)warp_sum(dF), Fs, dFs);
                if (!(dFs < 0.0)) break;
                const double step = newton_step(Fs, dFs, sparsemax);
                if (!(step > 1e-5 * fmax(1.0, fabs(tau)))) {  // the fp64 steps finish it
                    settled = step > -1e-5 * fmax(1.0, fabs(tau));
                    break;
                }
                tau += step;
                // pages with a + 8 b below the (rising) threshold contribute nothing any more
                if (!glob && (it & 3) == 3) {
                    int kept = 0;
                    for (int i0 = 0; i0 < cnt; i0 += 32) {
                        const int i = i0 + lane;
                        float ai = 0.f, bi = 0.f, ni = 0.f;
                        bool keep = false;
                        if (i < cnt) {
                            ai = xa[i]; bi = xb[i]; ni = xn[i];
                            keep = (double)ai + 8.0 * (double)bi > tau;
                        }
                        const unsigned bal = __ballot_sync(kFull, keep);
                        __syncwarp();
                        if (keep) {
                            const int pos = kept + __popc(bal & ((1u << lane) - 1u));
                            xa[pos] = ai; xb[pos] = bi; xn[pos] = ni;
                        }
                        kept += __popc(bal);
                        __syncwarp();
                    }
                    cnt = kept;
                }
            }
            // fp64 finish: the fp32 moments carry about 1e-7 relative error, which bounds how
            // close the fp32 iterates can get. Newton steps on double-precision moments over the
            // same survivors (pruned pages add below 1e-14 of their count) take the root to fp64
            // accuracy; each step squares the error, so from settled fp32 iterates (within about
            // 1e-5) two steps reach it.
#pragma unroll 1
            for (int it = 0; it < (settled ? 2 : 6); ++it) {
                double F = 0.0, dF = 0.0;
                if (!glob) {
                    for (int i = lane; i < cnt; i += 32) {
                        double E, dE;
                        trunc_moment_d(xa[i], xb[i], tau, sparsemax, E, dE);
                        F = fma((double)xn[i], E, F);
                        dF = fma((double)xn[i], dE, dF);
                    }
                } else {
                    for (int j = p0 + lane; j < p1; j += 32) {
                        float aj, bj;
                        double E, dE;
                        model(j, aj, bj);
                        trunc_moment_d(aj, bj, tau, sparsemax, E, dE);
                        F = fma((double)page_n(j), E, F);
                        dF = fma((double)page_n(j), dE, dF);
                    }
                }
                double Fs, dFs;
                reduce(warp_sum(F), warp_sum(dF), Fs, dFs);
                if (!(dFs < 0.0)) break;
                const double step = newton_step(Fs, dFs, sparsemax);
                tau += step;
                if (!(fabs(step) > 1e-13 * fmax(1.0, fabs(tau)))) break;
            }
            return tau;
        };
        double tau = 0.0;
        if (solo) {
            if (warp == 0)
                tau = newton(la, lb, ln, total, false, [&](double F, double dF, double &Fs, double &dFs) {
                    Fs = F;  // the warp's totals are the sums
                    dFs = dF;
                });
        } else {
            int ph = 0;  // parity of the partial-sum buffer of the next combine
            tau = newton(sa, sb, sn, cnt, cnt > capw, [&](double F, double dF, double &Fs, double &dFs) {
                // the warps' totals (double-buffered, one barrier), added in warp order
                if (lane == 0) { s_part[ph & 1][warp][0] = F; s_part[ph & 1][warp][1] = dF; }
                __syncthreads();
                Fs = 0.0;
                dFs = 0.0;
#pragma unroll
                for (int k = 0; k < NW; ++k) { Fs += s_part[ph & 1][k][0]; dFs += s_part[ph & 1][k][1]; }
                ++ph;
            });
        }
        if (tid == 0) {
            tau_hat[(size_t)b * H_q + hq] = (float)tau;
#pragma unroll
            for (int r = 0; r < G; ++r) st_dsmem_f64(dsmem(&s_tau[g], (uint32_t)r), tau);
        }
    }
    cluster_sync();  // every query's tau-hat has landed in every CTA

    // this CTA's slice of the union, ascending page order: warp w owns rows of 32 pages from
    // q0; a page's keep flags are computed once and kept as one bit word per row. The page
    // statistic is the bound UB, or (est_max) the Gaussian estimate of the page maximum capped
    // by the bound, min(UB, m + sqrt(2 ln n) sqrt(v)), decided in fp64.
    const float *ub0 = scores + ((size_t)b * H_q + h * G) * 3 * max_pages;
    double thr[G];
#pragma unroll
    for (int q = 0; q < G; ++q) thr[q] = s_tau[q] - (double)delta;
    const double zfull = est_max && P > 1 ? sqrt(2.0 * log((double)P)) : 0.0;
    // the page statistics of G queries for page j (rows past q1 read nothing)
    struct PageStats { float ub[G], m[G], v[G]; };
    auto load_page = [&](int j, bool in, PageStats &ps) {
#pragma unroll
        for (int q = 0; q < G; ++q) {
            const float *row = ub0 + (size_t)q * 3 * max_pages + j;
            ps.ub[q] = in ? __ldcg(row) : 0.f;
            ps.m[q] = in && est_max ? __ldcg(row + max_pages) : 0.f;
            ps.v[q] = in && est_max ? __ldcg(row + 2 * (size_t)max_pages) : 0.f;
        }
    };
    auto keep_page = [&](int j, const PageStats &ps) {
        bool keep = false;
        double zn = 0.0;
        if (est_max) {
            const int nj = len - j * P < P ? len - j * P : P;
            zn = nj == P ? zfull : (nj > 1 ? sqrt(2.0 * log((double)nj)) : 0.0);
        }
#pragma unroll
        for (int q = 0; q < G; ++q) {
            double x = (double)ps.ub[q];
            if (est_max) {
                const double e = (double)ps.m[q] + zn * sqrt(fmax((double)ps.v[q], 0.0));
                x = e < x ? e : x;
            }
            keep |= (double)am1 * x > thr[q];
        }
        return keep;
    };
    const int u0 = (int)((long long)n * g / G), u1 = (int)((long long)n * (g + 1) / G);
    const int per = ((u1 - u0 + NW - 1) / NW + 31) & ~31;
    const int q0 = min(u0 + warp * per, u1), q1 = min(q0 + per, u1);
    int mine = 0;
    for (int j0 = q0; j0 < q1; j0 += 64) {  // two rows of 32 pages, all their loads in flight
        const int ja = j0 + lane, jb = j0 + 32 + lane;
        PageStats sa_, sb_;
        load_page(ja, ja < q1, sa_);
        load_page(jb, jb < q1, sb_);
        const unsigned ba = __ballot_sync(kFull, ja < q1 && keep_page(ja, sa_));
        const unsigned bb = __ballot_sync(kFull, jb < q1 && keep_page(jb, sb_));
        if (lane == 0) {
            bits[(j0 - u0) >> 5] = ba;
            if (j0 + 32 < q1) bits[((j0 - u0) >> 5) + 1] = bb;
        }
        mine += __popc(ba) + __popc(bb);
    }
    if (lane == 0) s_cnt[warp] = mine;
    __syncthreads();
    int off = 0, slice = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        off += w < warp ? s_cnt[w] : 0;
        slice += s_cnt[w];
    }
    if (tid == 0) {
#pragma unroll
        for (int r = 0; r < G; ++r) st_dsmem_s32(dsmem(&s_kept[g], (uint32_t)r), slice);
    }
    cluster_sync();  // every slice's count has landed in every CTA
    int total = 0;
#pragma unroll
    for (int r = 0; r < G; ++r) {
        off += r < g ? s_kept[r] : 0;
        total += s_kept[r];
    }
    int32_t *out = sel_idx + (size_t)bh * max_sel;
    for (int j0 = q0; j0 < q1; j0 += 32) {
        const unsigned bal = bits[(j0 - u0) >> 5];
        const int at = off + __popc(bal & ((1u << lane) - 1u));
        if (((bal >> lane) & 1u) && at < max_sel) out[at] = j0 + lane;
        off += __popc(bal);
    }
    for (int j = total + g * NT + tid; j < max_sel; j += G * NT) out[j] = -1;
    if (g == 0 && tid == 0) {
        if (total > max_sel) flag(status, EKV_DEV_SEL_OVERFLOW);
        sel_count[bh] = total < max_sel ? total : max_sel;
    }
}

static cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, cudaStream_t st, bool pdl,
                                     cudaLaunchAttribute *attr)
{
    cudaLaunchConfig_t cfg = {};
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cfg;
}

cudaError_t launch_select_pages(const ekv_cache &c, int H_q, int policy, int topk, float alpha,
                                float delta, const float *scores, int32_t *sel_idx,
                                int32_t *sel_count, int max_sel, float *tau_hat, cudaStream_t st,
                                bool pdl)
{
    cudaLaunchAttribute attr[1];
    const dim3 grid(c.num_kv_heads, c.batch);
    if (policy == EKV_SEL_TOPK && c.max_pages <= 16 * kSelThreads) {
        // keys in registers: 8 or 16 per thread
        cudaLaunchConfig_t cfg = pdl_config(grid, dim3(kSelThreads), st, pdl, attr);
        if (c.max_pages <= 8 * kSelThreads)
            return cudaLaunchKernelEx(&cfg, select_topk_reg_kernel<8>, scores, c.num_kv_heads,
                                      c.max_pages, c.page_size, c.seq_lens, topk, sel_idx, sel_count,
                                      max_sel, c.dev_status);
        return cudaLaunchKernelEx(&cfg, select_topk_reg_kernel<16>, scores, c.num_kv_heads,
                                  c.max_pages, c.page_size, c.seq_lens, topk, sel_idx, sel_count,
                                  max_sel, c.dev_status);
    }
    if (policy == EKV_SEL_TOPK) {
        cudaLaunchConfig_t cfg = pdl_config(grid, dim3(kSelThreads), st, pdl, attr);
        const int keys = c.max_pages < kSmemKeys ? c.max_pages : kSmemKeys;
        cfg.dynamicSmemBytes = sizeof(uint32_t) * keys;
        static bool attr_set = false;
        if (!attr_set) {
            cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemKeys * (int)sizeof(uint32_t));
            attr_set = true;
        }
        return cudaLaunchKernelEx(&cfg, select_topk_kernel, scores, c.num_kv_heads, c.max_pages,
                                  c.page_size, c.seq_lens, topk, sel_idx, sel_count, max_sel,
                                  c.dev_status);
    }
    // one CTA per query, the G queries of a (sequence, KV head) in one cluster
    const int G = H_q / c.num_kv_heads;
    cudaLaunchAttribute gattr[2];
    gattr[0].id = cudaLaunchAttributeClusterDimension;
    gattr[0].val.clusterDim.x = G;
    gattr[0].val.clusterDim.y = 1;
    gattr[0].val.clusterDim.z = 1;
    gattr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    gattr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c.num_kv_heads * G, c.batch);
    cfg.blockDim = dim3(128);
    cfg.stream = st;
    cfg.attrs = gattr;
    cfg.numAttrs = pdl ? 2 : 1;
    // per-warp survivor capacity: a warp's whole page slice when the shared memory allows
    // slices | gathered list | one keep-bit word per 32 pages of a CTA's union slice
    const size_t bit_words = (size_t)(c.max_pages / G) / 32 + 16;
    const size_t fixed = sizeof(float) * 3 * kGaussList + sizeof(unsigned) * bit_words;
    if (fixed + 4 * 3 * sizeof(float) * 64 > (size_t)kGaussSmemBytes) return cudaErrorInvalidValue;
    const int cap_max = (int)(((size_t)kGaussSmemBytes - fixed) / (4 * 3 * sizeof(float))) & ~3;
    int capw = (c.max_pages + 3) / 4;
    capw = ((capw + 3) & ~3) < cap_max ? ((capw + 3) & ~3) : cap_max;
    cfg.dynamicSmemBytes = sizeof(float) * (size_t)4 * 3 * capw + fixed;
#define EKV_GSEL(GG)                                                                           \
    [&]() {                                                                                    \
        static bool attr_set = false;                                                          \
        if (!attr_set) {                                                                       \
            const cudaError_t e = cudaFuncSetAttribute(                                        \
                select_gauss_kernel<GG>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGaussSmemBytes); \
            if (e != cudaSuccess) return e;                                                    \
            attr_set = true;                                                                   \
        }                                                                                      \
        return cudaLaunchKernelEx(&cfg, select_gauss_kernel<GG>, scores, c.num_kv_heads,       \
                                  c.max_pages, c.page_size, c.seq_lens, alpha, delta, sel_idx, \
                                  sel_count, max_sel, tau_hat, c.dev_status, capw,             \
                                  policy == EKV_SEL_GAUSS_MAX);                                \
    }()
    switch (G) {
    case 1: return EKV_GSEL(1);
    case 2: return EKV_GSEL(2);
    case 4: return EKV_GSEL(4);
    default: return EKV_GSEL(8);
    }
#undef EKV_GSEL
}

}  // namespace ekv

namespace ekv {

// The kk largest of n scores S[0, n) (kk < n <= R * kSelThreads), key descending then index
// ascending, written to out[0, kk) in ascending index order: each thread holds R consecutive
// keys in registers and cta_topk decides.
template <int R>
__device__ void emit_topk_reg(const float *S, int n, int kk, TopkShared &ts, int32_t *out)
{
    constexpr int NT = kSelThreads;
    const int j0 = threadIdx.x * R;
    uint32_t u[R];
#pragma unroll
    for (int r = 0; r < R; ++r) u[r] = j0 + r < n ? topk_order_key(__ldcg(S + j0 + r)) : 0u;
    bool keep[R];
    const int mine = cta_topk<NT, R>(u, n, kk, ts, keep);
    int pos = block_incl_scan<NT>(mine, ts.warp_tot, nullptr) - mine;
#pragma unroll
    for (int r = 0; r < R; ++r)
        if (keep[r] && pos < kk) out[pos++] = j0 + r;
}

// Token-level top-T inside the selected pages, one 1024-thread CTA per (sequence, KV head).
// The candidate scores sit at slot i * P + t (selected page i, position t; -inf past a page's
// valid tokens); the exact radix select above keeps the T largest, ties to the lower slot, in
// slot order -- which is the candidate order (selection order, then position); up to 16384
// slots the keys are held in registers (emit_topk_reg). Emits
// (logical page, position) pairs, -1 padded to T, and the count.
__global__ void __launch_bounds__(kSelThreads)
select_tokens_kernel(const float *__restrict__ tscores, int H, int P, const int32_t *__restrict__ seq_lens,
                     int max_pages, const int32_t *__restrict__ sel_idx,
                     const int32_t *__restrict__ sel_count, int max_sel, int T,
                     int32_t *__restrict__ tok_page, int32_t *__restrict__ tok_pos,
                     int32_t *__restrict__ tok_count)
{
    constexpr int NT = kSelThreads;
    __shared__ int hist[2048];
    __shared__ int warp_tot[32];
    __shared__ int s_bin, s_above;
    __shared__ TopkShared ts;
    pdl_wait();
    const int tid = threadIdx.x;
    const int bh = blockIdx.x, b = bh / H;
    int ns = sel_count[bh];
    ns = ns < 0 ? 0 : (ns > max_sel ? max_sel : ns);
    int len;
    const int np = seq_pages(seq_lens, b, P, max_pages, nullptr, &len);
    const int32_t *sel = sel_idx + (size_t)bh * max_sel;
    // valid candidates: the tokens of the selected pages that exist
    int mine = 0;
    for (int i = tid; i < ns; i += NT) {
        const int j = sel[i];
        if (j >= 0 && j < np) mine += len - j * P < P ? len - j * P : P;
    }
    int n_valid;
    block_incl_scan<NT>(mine, warp_tot, &n_valid);
    const int n = ns * P;
    const float *S = tscores + (size_t)bh * max_sel * P;
    int32_t *pg = tok_page + (size_t)bh * T, *ps = tok_pos + (size_t)bh * T;
    int kk = T < n_valid ? T : n_valid;
    if (kk > 0) {
        if (kk == n_valid) {  // every valid candidate is kept: emit them in slot order
            int pos = 0;
            for (int j0 = 0; j0 < n; j0 += NT) {
                const int j = j0 + tid;
                const bool keep = j < n && __ldcg(S + j) > -INFINITY;
                int tot;
                const int incl = block_incl_scan<NT>(keep ? 1 : 0, warp_tot, &tot);
                if (keep && pos + incl - 1 < T) ps[pos + incl - 1] = j;
                pos += tot;
            }
            kk = pos < kk ? pos : kk;  // a non-finite score is not a candidate
        } else if (n <= 4 * NT) {
            emit_topk_reg<4>(S, n, kk, ts, ps);
        } else if (n <= 8 * NT) {
            emit_topk_reg<8>(S, n, kk, ts, ps);
        } else if (n <= 16 * NT) {
            emit_topk_reg<16>(S, n, kk, ts, ps);
        } else {
            radix_select_emit(n, kk, [&](int j) { return order_key(__ldcg(S + j)); }, hist, warp_tot,
                              &s_bin, &s_above, ps);
        }
    }
    __syncthreads();
    for (int k = tid; k < T; k += NT) {
        const int slot = k < kk ? ps[k] : -1;
        if (slot >= 0 && slot < n) {
            pg[k] = sel[slot / P];
            ps[k] = slot % P;
        } else {
            pg[k] = -1;
            ps[k] = -1;
        }
    }
    if (tid == 0) tok_count[bh] = kk;
    pdl_trigger();
}

cudaError_t launch_select_tokens(const ekv_cache &c, const float *tscores, const int32_t *sel_idx,
                                 const int32_t *sel_count, int max_sel, int T, int32_t *tok_page,
                                 int32_t *tok_pos, int32_t *tok_count, cudaStream_t st)
{
    select_tokens_kernel<<<c.batch * c.num_kv_heads, kSelThreads, 0, st>>>(
        tscores, c.num_kv_heads, c.page_size, c.seq_lens, c.max_pages, sel_idx, sel_count, max_sel,
        T, tok_page, tok_pos, tok_count);
    return cudaGetLastError();
}

}  // namespace ekv
