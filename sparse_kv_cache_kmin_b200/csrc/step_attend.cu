// step_attend.cu -- exact alpha-entmax attention over the selected pages with one thread-block
// cluster per (sequence, KV head) (EntmaxKV technical summary, §2.C: attention over the
// selected pages only; only the keys of those pages are read, and only the value rows that
// carry weight).
//
// The pages a (sequence, KV head) selected are split over the C CTAs of its cluster. A CTA
// resolves its pages (selection -> page table), then its 16 warps stream the K rows in 16-row
// tiles straight into registers (16 loads of 16 bytes in flight per lane, the load structure
// that reads scattered rows fastest), stage each tile in a per-warp shared-memory buffer with
// its 16-byte pieces XOR-swizzled by row, and take the logits of all G queries of the KV head
// with D / 16 warp-level bf16 MMAs (m16n8k16, fp32 accumulation). The logits z = (alpha-1) s
// stay in shared memory, with the maximum of every tile.
//
// The threshold tau solves sum_i [z_i - tau]_+^(1/(alpha-1)) = 1 over all the pair's tokens,
// which live in the cluster's distributed shared memory:
//   1. The tile maxima are logits, and the exact threshold of any subset of the logits is at
//      most tau (adding tokens only raises it). Each CTA reduces its own tile maxima to 64
//      group maxima per query and solves them exactly (cta_exact_tau): a lower bound on tau,
//      with no exchange yet.
//   2. Every token of the CTA above its bound is a candidate, listed in token order. One
//      cluster barrier; then every CTA reads all CTAs' bounds, largest logits and lists,
//      keeps the candidates above the largest bound, and -- up to 512 per query -- ranks each
//      against all the others, summing the values above it, which gives the closed-form
//      threshold of every support size at once (cta_exact_tau). More (nearly flat logits): an
//      fp64 bisection whose sums are reduced over the cluster, then the closed form over the
//      support it brackets.
//   3. Each CTA accumulates p_i v_i over its support tokens (V rows read only for those), in a
//      fixed order, and stores the sum into rank 0's shared memory; after a second cluster
//      barrier rank 0 adds the CTAs' partial outputs in rank order and writes the output.
#include "cluster.cuh"
#include "warp_entmax.cuh"  // closed_form_tau
#include "warp_mma.cuh"

namespace ekv {

constexpr int kAttThreads = 512;
constexpr int kAttWarps = kAttThreads / 32;
constexpr int kAttStageBytes = 8192;  // per warp: 16 loads of 16 bytes per lane
constexpr int kAttGroups = 64;        // lower-bound maxima per query over the cluster (2 per lane)
constexpr int kAttCand = 512;         // candidates the CTA solves by ranking
constexpr int kAttWarpSolve = 64;     // candidates one warp solves by sorting (2 per lane)

struct AttArgs {
    ekv_cache c;
    const void *q;
    int H_q;
    float qscale;  // scale * (alpha - 1)
    int sparsemax;
    const int32_t *sel_idx;
    const int32_t *sel_count;
    int max_sel;
    float *out;
    float *stat;
    int ent_cap;   // selected pages per CTA at most
};

// Small per-CTA state; the group maxima and candidate lists live in dynamic shared memory, on
// the tile staging buffers (free once the logits are taken).
template <int D, int G>
struct AttShared {
    // read by the cluster: this CTA's candidate count, largest logit and lower bound on tau
    int ccnt[G];
    float zmax_loc[G];
    double tlb_loc[G];
    int wcnt[kAttWarps];
    float zmax[G];               // the pair's largest logit
    double tlb[G];               // the pair's lower bound on tau (absolute)
    double tau[G];               // relative to zmax
    int fast[G];                 // 0: bisection, 1: solved by ranking (or no valid token)
    int best_k[G];
    int nset[G];                 // values per set handed to a solver
    int nbig[G];                 // values per set handed to the CTA-wide ranking solver
    int cnt_tab[G][17];          // candidate counts of every CTA, then their prefix
    float zm_tab[G][16];
    double tlb_tab[G][16];
    float part[kAttWarps];
    double fpart[2][G];          // bisection partial sums (read by the cluster)
    double cpart[3];             // closed-form partial sums (read by the cluster)
    double red[kAttWarps];
    float opart[kAttWarps][D];
};

__device__ __forceinline__ void st_shared_v4(void *p, const uint4 &v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_addr(p)), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// Exact thresholds of G small value sets at once, by the whole CTA. Set g holds n[g] values
// x = z - zmax <= 0 at vals[g * stride + i] (-inf entries are inert). Thread t serves set
// g = t / (NT / G) and its candidates i = t % (NT / G) + k NT / G: for each it counts the values
// above it (ties broken by index) and sums them and their squares in one short loop, which
// gives the closed-form threshold tau(k) of the support made of the k largest values. The
// threshold is tau(k) for the largest k with tau(k) <= x_(k) -- the sort-based rule of the
// oracle, evaluated for every k at once without a sort. A compact loop: the unrolled
// single-warp sorting networks it replaces ran from a cold instruction cache. tau[g] is
// written in fp64 (sums in fp32: values in [-1, 0], at most a few hundred of them).
template <int NT, int G>
__device__ void cta_exact_tau(const float *vals, int stride, const int *n, bool sparsemax,
                              double *tau, int *best_k)
{
    constexpr int TPG = NT / G;
    const int tid = threadIdx.x, g = tid / TPG, it = tid - g * TPG;
    if (tid < G) best_k[tid] = 0;
    __syncthreads();
    const int ng = n[g];
    const float *v = vals + (size_t)g * stride;
    int best = 0;
    float best_t = 0.f;
    for (int i = it; i < ng; i += TPG) {
        const float x = v[i];
        if (!(x > -INFINITY)) continue;
        float s1 = x, s2 = x * x;
        int rank = 0;
        auto visit = [&](float y, int j) {
            const bool before = y > x || (y == x && j < i);
            rank += before;
            s1 += before ? y : 0.f;
            s2 += before ? y * y : 0.f;
        };
        int j = 0;
        for (; j + 4 <= ng; j += 4) {  // four values per shared-memory load (vals is 16-byte aligned)
            const float4 y = *reinterpret_cast<const float4 *>(v + j);
            visit(y.x, j);
            visit(y.y, j + 1);
            visit(y.z, j + 2);
            visit(y.w, j + 3);
        }
        for (; j < ng; ++j) visit(v[j], j);
        const int k = rank + 1;
        const float kf = (float)k;
        float tk;
        bool ok = true;
        if (sparsemax) {
            tk = (s1 - 1.0f) / kf;
        } else {
            const float mean = s1 / kf;
            const float disc = (1.0f - fmaxf(s2 - s1 * mean, 0.f)) / kf;
            ok = disc >= 0.f;
            tk = mean - sqrtf(fmaxf(disc, 0.f));
        }
        if (ok && tk <= x && k > best) {
            best = k;
            best_t = tk;
        }
    }
    if (best > 0) atomicMax(&best_k[g], best);
    __syncthreads();
    if (best > 0 && best == best_k[g]) tau[g] = (double)best_t;  // k is unique within a set
    __syncthreads();
}

template <int D, int G>
__global__ void __launch_bounds__(kAttThreads, 1)
step_attend_kernel(AttArgs a)
{
    constexpr int NT = kAttThreads, NW = kAttWarps;
    constexpr int RB = D * 2;                 // bytes per bf16 row
    constexpr int W = RB / 16;                // 16-byte pieces per row
    constexpr int TB = 16 * RB;               // bytes per 16-row tile
    constexpr int TPL = TB / 512;             // pieces per lane per tile
    constexpr int TPS = kAttStageBytes / TB;  // tiles per warp step
    constexpr int KS = D / 16;                // MMA k-steps per tile
    static_assert(G <= 8, "one n = 8 MMA column block");
    static_assert(G * (3 * kAttCand + 16 * D) * 4 <= kAttWarps * kAttStageBytes,
                  "the lists and partial outputs fit on the staging buffers");
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ AttShared<D, G> sh;

    const ekv_cache &c = a.c;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_rank(), C = cluster_size();
    const int H = c.num_kv_heads, P = c.page_size, TPP = P / 16;
    const int bh = blockIdx.x / (int)C, b = bh / H, h = bh % H;
    const int ent_cap = a.ent_cap, ntok_cap = ent_cap * P, tile_cap = ent_cap * TPP;
    unsigned char *stage = smem + (size_t)warp * kAttStageBytes;
    float *zs = reinterpret_cast<float *>(smem + (size_t)NW * kAttStageBytes);  // [G][ntok_cap]
    int *ent_blk = reinterpret_cast<int *>(zs + (size_t)G * ntok_cap);        // [ent_cap]
    int *ent_nt = ent_blk + ent_cap;                                            // [ent_cap]
    float *tmax = reinterpret_cast<float *>(ent_nt + ent_cap);                  // [G][tile_cap]
    // after the logits phase, on the staging buffers:
    float *cx = reinterpret_cast<float *>(smem);                 // [G][kAttCand] candidate logits (cluster-read)
    int *ct = reinterpret_cast<int *>(cx + G * kAttCand);        // [G][kAttCand] their tokens
    float *gat = reinterpret_cast<float *>(ct + G * kAttCand);   // [G][kAttCand] values to solve
    float *oall = gat + G * kAttCand;                            // rank 0: [C][G][D] partial outputs

    pdl_wait();
    int len;
    const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
    int ns = a.sel_count[bh];
    ns = ns < 0 ? 0 : (ns > a.max_sel ? a.max_sel : ns);
    const int e0 = (int)((long long)ns * rank / C), e1 = (int)((long long)ns * (rank + 1) / C);
    for (int i = tid; i < e1 - e0; i += NT) {
        // entry i of this CTA: selected page j -> its block and valid tokens
        const int j = a.sel_idx[(size_t)bh * a.max_sel + e0 + i];
        int blk = -1, nt = 0;
        if (j < 0 || j >= np) {
            flag(c.dev_status, EKV_DEV_BAD_SEL);
        } else {
            const int bk = c.page_table[(size_t)b * c.max_pages + j];
            if (bk < 0 || bk >= c.num_blocks) {
                flag(c.dev_status, EKV_DEV_BAD_BLOCK);
            } else {
                blk = bk;
                nt = len - j * P < P ? len - j * P : P;
            }
        }
        ent_blk[i] = blk;
        ent_nt[i] = nt;
    }
    const int ne = e1 - e0, ntiles = ne * TPP, ntok = ne * P;
    if (tid < G) sh.ccnt[tid] = 0;
    // B fragments of the group's queries: column n = lane / 4 is query n (zero past G)
    uint32_t qb[KS][2];
    {
        const int n = lane >> 2;
        const uint32_t *qr = reinterpret_cast<const uint32_t *>(
            static_cast<const char *>(a.q) + (((size_t)b * a.H_q + (size_t)h * G + (n < G ? n : 0)) * D) * 2);
#pragma unroll
        for (int s = 0; s < KS; ++s) {
            qb[s][0] = n < G ? __ldg(qr + s * 8 + (lane & 3)) : 0u;
            qb[s][1] = n < G ? __ldg(qr + s * 8 + 4 + (lane & 3)) : 0u;
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- logits
    const char *kc = static_cast<const char *>(c.k_cache);
    const int lrow = lane & 15, lk = lane >> 4;
    const int r0 = lane >> 2, n0 = (lane & 3) * 2;
    for (int t0 = warp * TPS; t0 < ntiles; t0 += NW * TPS) {
        uint4 x[TPS][TPL];
        int ntt[TPS];
#pragma unroll
        for (int u = 0; u < TPS; ++u) {
            const int t = t0 + u;
            const int e = t / TPP, sub = t - e * TPP;
            const int blk = t < ntiles ? ent_blk[e] : -1;
            ntt[u] = blk >= 0 ? ent_nt[e] - sub * 16 : 0;
            const char *g = kc + (((size_t)(blk < 0 ? 0 : blk) * H + h) * P + sub * 16) * RB;
#pragma unroll
            for (int k = 0; k < TPL; ++k)
                x[u][k] = ntt[u] > 0 ? ld_stream16(g + (k * 32 + lane) * 16) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < TPS; ++u)
#pragma unroll
            for (int k = 0; k < TPL; ++k) {
                const int p = k * 32 + lane, row = p / W, pc = p % W;
                st_shared_v4(stage + u * TB + row * RB + ((pc ^ (row & 7)) << 4), x[u][k]);
            }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < TPS; ++u) {
            const int t = t0 + u;
            if (t >= ntiles) break;  // uniform over the warp
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const unsigned char *tile = stage + u * TB;
#pragma unroll
            for (int s = 0; s < KS; ++s) {
                uint32_t af[4];
                const int pc = s * 2 + lk;
                ldsm_x4(af, tile + lrow * RB + ((pc ^ (lrow & 7)) << 4));
                mma_bf16_16816(acc, af, qb[s][0], qb[s][1]);
            }
            const float z00 = r0 < ntt[u] ? a.qscale * acc[0] : -INFINITY;
            const float z01 = r0 < ntt[u] ? a.qscale * acc[1] : -INFINITY;
            const float z10 = r0 + 8 < ntt[u] ? a.qscale * acc[2] : -INFINITY;
            const float z11 = r0 + 8 < ntt[u] ? a.qscale * acc[3] : -INFINITY;
            const int tok = t * 16 + r0;
            float m0 = fmaxf(z00, z10), m1 = fmaxf(z01, z11);
            if (n0 < G) {
                zs[(size_t)n0 * ntok_cap + tok] = z00;
                zs[(size_t)n0 * ntok_cap + tok + 8] = z10;
            }
            if (n0 + 1 < G) {
                zs[(size_t)(n0 + 1) * ntok_cap + tok] = z01;
                zs[(size_t)(n0 + 1) * ntok_cap + tok + 8] = z11;
            }
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                m0 = fmaxf(m0, __shfl_xor_sync(kFull, m0, o));
                m1 = fmaxf(m1, __shfl_xor_sync(kFull, m1, o));
            }
            if (lane < 4 && n0 < G) tmax[(size_t)n0 * tile_cap + t] = m0;
            if (lane < 4 && n0 + 1 < G) tmax[(size_t)(n0 + 1) * tile_cap + t] = m1;
        }
        __syncwarp();  // the stage is read before the next tiles overwrite it
    }
    __syncthreads();

    // ---------------------------------------------------------------- local lower bound on tau
    // The tile maxima are logits, and the threshold of any subset of the logits is at most tau
    // (adding tokens only raises it). Each query's tiles in this CTA are grouped into
    // kAttGroups runs; one warp per query sorts the runs' maxima and solves them exactly, which
    // bounds the pair's tau from below with no exchange.
    {
        static_assert(G * kAttGroups <= NT && kAttGroups == 64, "one maximum per thread, two per lane");
        float x = -INFINITY;
        if (tid < G * kAttGroups) {
            const int g = tid / kAttGroups, k = tid - g * kAttGroups;
            const int ta = (int)((long long)ntiles * k / kAttGroups);
            const int tb = (int)((long long)ntiles * (k + 1) / kAttGroups);
            for (int t = ta; t < tb; ++t) x = fmaxf(x, tmax[(size_t)g * tile_cap + t]);
            gat[tid] = x;
        }
        __syncthreads();
        if (warp < G) {
            const int g = warp;
            float v[2] = {gat[g * kAttGroups + lane], gat[g * kAttGroups + 32 + lane]};
            const float zm = warp_max(fmaxf(v[0], v[1]));
            double lb = -INFINITY;
            if (zm > -INFINITY) {
                v[0] -= zm;  // -inf stays -inf
                v[1] -= zm;
                const int cnt = __popc(__ballot_sync(kFull, v[0] > -INFINITY)) +
                                __popc(__ballot_sync(kFull, v[1] > -INFINITY));
                const double t = warp_exact_tau<2>(v, cnt, a.sparsemax != 0);
                // lowered a little so that fp32 rounding never drops a support member
                lb = (double)zm + t - 1e-5 * fmax(1.0, fabs(t));
            }
            if (lane == 0) {
                sh.zmax_loc[g] = zm;
                sh.tlb_loc[g] = lb;
            }
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- local candidates, token order
    {
        constexpr int WPQ = NW / G;  // warps per query
        const int g = warp % G, part = warp / G;
        const int ta = (int)((long long)ntok * part / WPQ), tb = (int)((long long)ntok * (part + 1) / WPQ);
        const float *zg = zs + (size_t)g * ntok_cap;
        const double lb = sh.tlb_loc[g];
        int mine = 0;
        for (int i = ta + lane; i - lane < tb; i += 32)
            mine += __popc(__ballot_sync(kFull, i < tb && (double)zg[i] > lb));
        if (lane == 0) sh.wcnt[warp] = mine;
        __syncthreads();
        int pos = 0;
        for (int p = 0; p < part; ++p) pos += sh.wcnt[p * G + g];
        for (int i = ta + lane; i - lane < tb; i += 32) {
            const float z = i < tb ? zg[i] : -INFINITY;
            const bool keep = i < tb && (double)z > lb;
            const unsigned bal = __ballot_sync(kFull, keep);
            const int at = pos + __popc(bal & ((1u << lane) - 1u));
            if (keep && at < kAttCand) {
                cx[g * kAttCand + at] = z;
                ct[g * kAttCand + at] = i;
            }
            pos += __popc(bal);
        }
        if (part == WPQ - 1 && lane == 0) sh.ccnt[g] = pos;
    }
    cluster_sync();

    // ---------------------------------------------------------------- exact tau
    // every CTA's count, largest logit and bound; the pair's bound is the largest of them
    if (tid < G * (int)C) {
        const int g = tid / C, cr = tid - g * C;
        sh.cnt_tab[g][cr + 1] = ld_dsmem(dsmem(&sh.ccnt[g], (uint32_t)cr));
        sh.zm_tab[g][cr] = ld_dsmem_f32(dsmem(&sh.zmax_loc[g], (uint32_t)cr));
        sh.tlb_tab[g][cr] = ld_dsmem_f64(dsmem(&sh.tlb_loc[g], (uint32_t)cr));
    }
    __syncthreads();
    if (tid < G) {  // prefix over the CTAs; a list that overflowed sends the query to bisection
        int run = 0;
        bool each_fits = true;
        float zm = -INFINITY;
        double lb = -INFINITY;
        sh.cnt_tab[tid][0] = 0;
        for (uint32_t cr = 0; cr < C; ++cr) {
            const int n = sh.cnt_tab[tid][cr + 1];
            zm = fmaxf(zm, sh.zm_tab[tid][cr]);
            lb = fmax(lb, sh.tlb_tab[tid][cr]);
            each_fits = each_fits && n <= kAttCand;
            run += n;
            sh.cnt_tab[tid][cr + 1] = run;
        }
        const bool solve = zm > -INFINITY && each_fits && run <= kAttCand;
        sh.zmax[tid] = zm;
        sh.tlb[tid] = lb;
        sh.nset[tid] = solve ? run : 0;
        sh.fast[tid] = zm == -INFINITY || solve;
        sh.tau[tid] = 0.0;
    }
    __syncthreads();
    // every query's candidates above the pair's bound, in cluster-wide token order, then one
    // ranking solve for all (values below the bound enter as -inf, which the solver skips)
    {
        // all of a thread's remote loads in flight together, then the stores
        static_assert((G * kAttCand) % NT == 0, "whole rounds");
        constexpr int PER = G * kAttCand / NT;
        float zv[PER];
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int i = tid + k * NT, g = i / kAttCand, idx = i - g * kAttCand;
            zv[k] = -INFINITY;
            if (idx < sh.nset[g]) {
                uint32_t cr = 0;
                while (idx >= sh.cnt_tab[g][cr + 1]) ++cr;
                zv[k] = ld_dsmem_f32(dsmem(&cx[g * kAttCand + idx - sh.cnt_tab[g][cr]], cr));
            }
        }
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int i = tid + k * NT, g = i / kAttCand, idx = i - g * kAttCand;
            if (idx < sh.nset[g]) gat[i] = (double)zv[k] > sh.tlb[g] ? zv[k] - sh.zmax[g] : -INFINITY;
        }
    }
    __syncthreads();
    {
        // up to kAttWarpSolve candidates: one warp per query sorts them (no barrier); more: the
        // CTA-wide ranking solve
        bool big = false;
#pragma unroll
        for (int gg = 0; gg < G; ++gg) big = big || sh.nset[gg] > kAttWarpSolve;  // the same in every thread
        if (warp < G && sh.nset[warp] > 0 && sh.nset[warp] <= kAttWarpSolve) {
            constexpr int RW = kAttWarpSolve / 32;
            const int g = warp, n = sh.nset[g];
            float v[RW];
            int cnt = 0;
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const int e = r * 32 + lane;
                v[r] = e < n ? gat[g * kAttCand + e] : -INFINITY;
                cnt += __popc(__ballot_sync(kFull, v[r] > -INFINITY));
            }
            const double t = warp_exact_tau<RW>(v, cnt, a.sparsemax != 0);
            if (lane == 0) sh.tau[g] = t;
        }
        if (big) {
            if (tid < G) sh.nbig[tid] = sh.nset[tid] > kAttWarpSolve ? sh.nset[tid] : 0;
            cta_exact_tau<NT, G>(gat, kAttCand, sh.nbig, a.sparsemax != 0, sh.tau, sh.best_k);
        }
    }
    // Too many candidates for the ranking solve (nearly flat logits): fp64 bisection on
    // f(t) = sum [x - t]_+^p over the cluster's tokens, then the closed form over the support
    // it brackets. The decision is the same in every CTA (the same counts were read), so every
    // CTA takes the same cluster barriers.
    for (int g = 0; g < G; ++g) {
        if (sh.fast[g] != 0) continue;
        const float zm = sh.zmax[g];
        const float *zg = zs + (size_t)g * ntok_cap;
        double lo = sh.tlb[g] - (double)zm, hi = 0.0;
        auto cluster_total = [&](double v, double *slot) {  // sum over the cluster, rank order
            v = warp_sum(v);
            if (lane == 0) sh.red[warp] = v;
            __syncthreads();
            if (tid == 0) {
                double s = 0.0;
                for (int w = 0; w < NW; ++w) s += sh.red[w];
                *slot = s;
            }
            cluster_sync();
            double tot = 0.0;
            for (uint32_t cr = 0; cr < C; ++cr) tot += ld_dsmem_f64(dsmem(slot, cr));
            return tot;
        };
        for (int it = 0; it < 60; ++it) {
            const double mid = 0.5 * (lo + hi);
            double f = 0.0;
            for (int i = tid; i < ntok; i += NT) {
                const double r = (double)(zg[i] - zm) - mid;
                if (r > 0.0) f += a.sparsemax ? r : r * r;
            }
            const double F = cluster_total(f, &sh.fpart[it & 1][g]);
            if (F >= 1.0) lo = mid; else hi = mid;
        }
        double s1 = 0.0, s2 = 0.0, k = 0.0;
        for (int i = tid; i < ntok; i += NT) {
            const double x = (double)(zg[i] - zm);
            if (x > lo) { s1 += x; s2 += x * x; k += 1.0; }
        }
        s1 = cluster_total(s1, &sh.cpart[0]);
        s2 = cluster_total(s2, &sh.cpart[1]);
        k = cluster_total(k, &sh.cpart[2]);
        double tau = lo;
        if (k > 0.0) closed_form_tau(k, s1, s2, a.sparsemax != 0, tau);
        __syncthreads();
        if (tid == 0) sh.tau[g] = tau;
        cluster_sync();  // every CTA has read the partial sums before they are reused
    }
    __syncthreads();

    // ---------------------------------------------------------------- output
    // p_i v_i over this CTA's support tokens (V rows read only for those), summed over the
    // CTA's warps in a fixed order and pushed into rank 0's shared memory; rank 0 adds the CTAs'
    // partial outputs in rank order.
    {
        constexpr int WPQ = NW / G;
        const int g = warp % G, part = warp / G;
        const float zm = sh.zmax[g];
        const double tau = sh.tau[g];
        const int half = lane >> 4, hl = lane & 15;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        const char *vc = static_cast<const char *>(c.v_cache);
        auto add_row = [&](int tl, double r) {
            const float p = (float)(a.sparsemax ? r : r * r);
            const int e = tl / P, tok = tl - e * P;
            const int blk = ent_blk[e];
            if (hl < W && blk >= 0) {
                const uint4 v = ld_stream16(vc + (((size_t)blk * H + h) * P + tok) * RB + hl * 16);
                float f[8];
                Chunk<EKV_BF16>::unpack(v, f);
#pragma unroll
                for (int q8 = 0; q8 < 8; ++q8) acc[q8] = fmaf(p, f[q8], acc[q8]);
            }
        };
        if (zm > -INFINITY) {
            if (sh.fast[g] != 0) {
                // this CTA's candidates (<= kAttCand on this path); a half-warp takes rows
                // i, i + 2 WPQ, ... and keeps up to four value-row loads in flight
                const int n = sh.ccnt[g];
                constexpr int RF = 4;
                for (int i0 = part * 2 + half; i0 < n; i0 += RF * WPQ * 2) {
                    uint4 vv[RF];
                    float pr[RF];
#pragma unroll
                    for (int u = 0; u < RF; ++u) {
                        const int i = i0 + u * WPQ * 2;
                        pr[u] = 0.f;
                        vv[u] = make_uint4(0, 0, 0, 0);
                        if (i < n) {
                            const double r = (double)(cx[g * kAttCand + i] - zm) - tau;
                            const int tl = ct[g * kAttCand + i], e = tl / P, blk = ent_blk[e];
                            if (r > 0.0 && blk >= 0) {
                                pr[u] = (float)(a.sparsemax ? r : r * r);
                                if (hl < W)
                                    vv[u] = ld_stream16(vc + (((size_t)blk * H + h) * P + (tl - e * P)) * RB + hl * 16);
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < RF; ++u) {
                        float f[8];
                        Chunk<EKV_BF16>::unpack(vv[u], f);
#pragma unroll
                        for (int q8 = 0; q8 < 8; ++q8) acc[q8] = fmaf(pr[u], f[q8], acc[q8]);
                    }
                }
            } else {
                const float *zg = zs + (size_t)g * ntok_cap;
                for (int i = part * 2 + half; i < ntok; i += WPQ * 2) {
                    const double r = (double)(zg[i] - zm) - tau;
                    if (r > 0.0) add_row(i, r);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(kFull, acc[e], 16);
        if (half == 0 && hl < W) {
#pragma unroll
            for (int e = 0; e < 8; ++e) sh.opart[warp][hl * 8 + e] = acc[e];
        }
        __syncthreads();
        for (int i = tid; i < G * D; i += NT) {
            const int gg = i / D, dd = i - gg * D;
            float s = 0.f;
            for (int p = 0; p < WPQ; ++p) s += sh.opart[p * G + gg][dd];
            st_dsmem_f32(dsmem(&oall[(size_t)rank * G * D + i], 0u), s);
        }
    }
    cluster_sync();  // the partial outputs have landed; no CTA's shared memory is read after this
    if (rank == 0) {
        const size_t bq0 = (size_t)b * a.H_q + (size_t)h * G;
        for (int i = tid; i < G * D; i += NT) {
            float s = 0.f;
            for (uint32_t cr = 0; cr < C; ++cr) s += oall[(size_t)cr * G * D + i];
            a.out[bq0 * D + i] = s;
        }
        if (tid < G)
            a.stat[bq0 + tid] = sh.zmax[tid] == -INFINITY ? -INFINITY : (float)((double)sh.zmax[tid] + sh.tau[tid]);
    }
    pdl_trigger();
}

// Dynamic shared memory of the kernel for `ent_cap` pages per CTA.
static size_t att_smem_bytes(int ent_cap, int P, int G)
{
    const size_t ntok = (size_t)ent_cap * P, tiles = (size_t)ent_cap * (P / 16);
    return (size_t)kAttWarps * kAttStageBytes + sizeof(float) * G * ntok + 2 * sizeof(int) * ent_cap +
           sizeof(float) * G * tiles;
}

template <int D, int G>
static cudaError_t launch_attend_t(const AttArgs &a0, cudaStream_t st, bool pdl, bool *launched)
{
    auto k = step_attend_kernel<D, G>;
    const ekv_cache &c = a0.c;
    *launched = false;
    int dev = 0, sms = 148, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    // the kernel's own static shared memory, as compiled, bounds the dynamic part
    static size_t stat_bytes = 0;  // per instantiation
    static bool attr_set = false, attr_ok = false;
    if (!attr_set) {
        attr_set = true;
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, k) == cudaSuccess && (size_t)optin > fa.sharedSizeBytes) {
            stat_bytes = fa.sharedSizeBytes;
            attr_ok = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)((size_t)optin - stat_bytes)) == cudaSuccess &&
                      cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
        }
        if (!attr_ok) cudaGetLastError();  // not served; leave no error behind for later calls
    }
    if (!attr_ok) return cudaSuccess;
    const size_t dyn_max = (size_t)optin - stat_bytes;
    const int pairs = c.batch * c.num_kv_heads;
    int C = 1;
    while (C < 16 && (long long)pairs * C * 2 <= sms) C *= 2;
    auto smem_for = [&](int Cc) { return att_smem_bytes((a0.max_sel + Cc - 1) / Cc, c.page_size, G); };
    while (C <= 16 && smem_for(C) > dyn_max) C *= 2;
    // not served (the caller takes the chunk kernels): a selection too large for 16 CTAs, or
    // clusters that would not all be resident at once
    if (C > 16 || (C > 1 && (long long)pairs * C > sms)) return cudaSuccess;
    AttArgs a = a0;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kAttThreads);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    auto set_c = [&](int Cc) {
        a.ent_cap = (a0.max_sel + Cc - 1) / Cc;
        attr[0].val.clusterDim.x = Cc;
        cfg.gridDim = dim3((unsigned)(pairs * Cc));
        cfg.dynamicSmemBytes = smem_for(Cc);
    };
    set_c(C);
    // a smaller cluster when the GPU cannot hold every cluster of this size at once
    for (;;) {
        int active = 0;
        if (cudaOccupancyMaxActiveClusters(&active, (const void *)k, &cfg) != cudaSuccess) {
            cudaGetLastError();
            active = 0;
        }
        const int Cn = C / 2;
        if (active >= pairs || Cn < 1 || smem_for(Cn) > dyn_max) break;
        C = Cn;
        set_c(C);
    }
    *launched = true;
    return cudaLaunchKernelEx(&cfg, k, a);
}

// Launches the cluster attention when it serves the call (bf16, entmax, P a multiple of 16,
// d in {64, 128}, G <= 8, the selection fits the cluster's shared memory); otherwise launches
// nothing and leaves *launched false.
cudaError_t launch_step_attend(const ekv_cache &c, const void *q, int H_q, float scale, int attn,
                               const int32_t *sel_idx, const int32_t *sel_count, int max_sel,
                               float *out, float *stat, cudaStream_t st, bool pdl, bool *launched)
{
    *launched = false;
    if (c.dtype != EKV_BF16 || attn == EKV_SOFTMAX || c.page_size % 16 != 0) return cudaSuccess;
    AttArgs a;
    a.c = c;
    a.q = q;
    a.H_q = H_q;
    const float alpha = attn == EKV_ENTMAX15 ? 1.5f : 2.0f;
    a.qscale = scale * (alpha - 1.0f);
    a.sparsemax = attn == EKV_SPARSEMAX;
    a.sel_idx = sel_idx;
    a.sel_count = sel_count;
    a.max_sel = max_sel;
    a.out = out;
    a.stat = stat;
    a.ent_cap = max_sel;
    const int G = H_q / c.num_kv_heads;
    if (c.head_dim == 128) {
        switch (G) {
        case 1: return launch_attend_t<128, 1>(a, st, pdl, launched);
        case 2: return launch_attend_t<128, 2>(a, st, pdl, launched);
        case 4: return launch_attend_t<128, 4>(a, st, pdl, launched);
        default: return launch_attend_t<128, 8>(a, st, pdl, launched);
        }
    }
    switch (G) {
    case 1: return launch_attend_t<64, 1>(a, st, pdl, launched);
    case 2: return launch_attend_t<64, 2>(a, st, pdl, launched);
    case 4: return launch_attend_t<64, 4>(a, st, pdl, launched);
    default: return launch_attend_t<64, 8>(a, st, pdl, launched);
    }
}

}  // namespace ekv
