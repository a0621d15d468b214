// decode.cu -- attention over the selected pages only (EntmaxKV technical summary, §2.C),
// read in place from the paged cache: no gather copy, no dense materialisation.
//
// Two kernels per call.
//
// decode_chunk_kernel: the selected pages of each (sequence, KV head) are cut into chunks of
// CP pages (CP * P <= 256 tokens); a persistent grid walks the flattened (chunk, sequence,
// head) list. For a chunk, the eight warps stream the K rows of its pages (a row of d
// elements is W = d * size / 16 lanes of 16-byte loads; each lane keeps four rows in flight
// and holds the matching 16-byte slice of the G group queries, pre-scaled, in registers),
// reduce the per-row partial dots with a transposing butterfly and leave the G x (CP * P)
// logits in shared memory.
//   softmax: p = 2^(z - m) with the chunk max m, l = sum p, then the same warps stream the V
//            rows and accumulate sum p v; the chunk writes (m, l, sum p v) -- the usual
//            log-sum-exp partial.
//   entmax:  the chunk writes its logits z = (alpha-1) * scale * q.k and its max to the
//            workspace; no V is read yet, because most V rows carry zero weight.
//
// decode_finish_kernel, one CTA per (sequence, query head):
//   softmax: merges the chunk partials with the log-sum-exp rule.
//   entmax:  the threshold satisfies tau >= max z - 1 (the largest weight is at most 1), so
//            only logits above max z - 1 can be in the support. The CTA gathers them,
//            runs Newton's method on f(tau) = sum [z - tau]_+^(1/(alpha-1)) - 1 (convex,
//            decreasing, so from the left it climbs monotonically to the root), then fixes
//            the support S = {z > tau} and recomputes tau in closed form over S in fp64
//            (sparsemax: (sum_S z - 1) / |S|; 1.5-entmax: mean_S - sqrt((1 - sum_S (z -
//            mean_S)^2) / |S|)), repeating until S is stable. Only the V rows of S are read.
#include "decode.cuh"
#include "warp_entmax.cuh"

namespace ekv {

constexpr int kNW = 8;         // consumer warps per CTA
constexpr int kThreads = (kNW + 1) * 32;

// Tokens per chunk: a K tile (entmax) or a K + V tile (softmax) of about 32 KiB per pipeline
// stage, at least one page, at most 256 tokens, a whole number of pages.
__host__ __device__ constexpr int chunk_tokens(int row_bytes, int P, bool softmax)
{
    int t = (softmax ? 16384 : 32768) / row_bytes;
    t = t > 256 ? 256 : t;
    t = (t / P) * P;
    return t < P ? P : t;
}

constexpr int kStages = 3;  // pipeline depth (shared-memory stages per CTA)

// Bytes of one pipeline stage: the group's query rows (rounded to 128 B), then the K tile
// (and the V tile for softmax).
__host__ __device__ constexpr int stage_q_bytes(int G, int D, int esz) { return (G * D * esz + 127) / 128 * 128; }

// Producer/consumer pipeline over the flattened (chunk, sequence, KV head) items of a
// persistent grid. Warp kNW (the producer) walks the CTA's items, skips empty ones, resolves
// the next item's pages (selection -> page table, validated) while the previous copies are in
// flight, then waits for a free stage and issues one bulk copy per page span -- K rows, and V
// rows for softmax -- plus one for the group's query rows, all completing on the stage's
// `full` barrier. The eight consumer warps wait on `full`, compute from shared memory and
// release the stage through its `empty` barrier. Every wait is bounded by the global timer:
// on expiry the kernel flags EKV_DEV_TIMEOUT and stops.
template <int DT, int D, int G, bool SOFTMAX>
__global__ void __launch_bounds__(kThreads)
decode_chunk_kernel(DecodeArgs a)
{
    constexpr int EPC = Chunk<DT>::N;
    constexpr int ESZ = Chunk<DT>::kBytes;
    constexpr int RB = D * ESZ;      // bytes per token row
    constexpr int W = RB / 16;       // lanes per token row
    constexpr int RPI = 32 / W;      // rows per warp instruction
    constexpr int TPL = 4;           // rows per lane per step
    constexpr int TW = TPL * RPI;    // rows per warp step
    constexpr int NQK = TPL * G;
    constexpr int OUTN = NQK >= W ? NQK / W : 1;
    constexpr int QB = stage_q_bytes(G, D, ESZ);
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t bar_full[kStages], bar_empty[kStages];
    __shared__ int blk_s[kStages][kMaxCP], ntok_s[kStages][kMaxCP];
    __shared__ long long item_s[kStages];
    __shared__ float m_s[G], l_s[G];
    __shared__ int ok_s;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const ekv_cache &c = a.c;
    const int H = c.num_kv_heads, P = c.page_size, BH = c.batch * H;
    const int CT = a.CP * P;                         // tokens per chunk
    const int stage_bytes = QB + CT * RB * (SOFTMAX ? 2 : 1);
    unsigned char *stage0 = smem;
    const int NS = a.stages;
    float *z_s = reinterpret_cast<float *>(smem + NS * stage_bytes);        // [G][CT]
    float *o_s = z_s + G * CT;                                              // softmax: [kNW][G][D]
    const long long items = (long long)BH * a.NC;

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&bar_full[i], 1);
            mbar_init(&bar_empty[i], kNW * 32);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();

    if (warp == kNW) {
        // ------------------------------------------------------------------ producer
        const char *kc = static_cast<const char *>(c.k_cache);
        const char *vc = static_cast<const char *>(c.v_cache);
        const char *qc = static_cast<const char *>(a.q);
        // the next non-empty item at or after `it`, with this lane's page of it resolved
        long long it = blockIdx.x;
        int ci = 0, bh = 0, blk = 0, nt = 0;
        auto advance = [&]() {
            int nsel = 0;
            for (; it < items; it += gridDim.x) {
                ci = (int)(it / BH);
                bh = (int)(it % BH);
                nsel = a.sel_count[bh];
                nsel = nsel < 0 ? 0 : (nsel > a.max_sel ? a.max_sel : nsel);
                if (ci * a.CP < nsel) break;
            }
            blk = 0;
            nt = 0;
            if (it >= items || lane >= a.CP) return;
            const int b = bh / H;
            int len;
            const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
            const int i = ci * a.CP + lane;
            if (i < nsel) {
                const int j = a.sel_idx[(size_t)bh * a.max_sel + i];
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
                if (!SOFTMAX) a.sel_blk[(size_t)bh * a.max_sel + i] = nt > 0 ? blk : -1;
            }
        };
        advance();
        for (int k = 0;; ++k) {
            const int buf = k % NS;
            const uint32_t ph = (k / NS) & 1;
            int free_ok = lane == 0 ? (int)mbar_wait_bounded(&bar_empty[buf], ph ^ 1) : 0;
            free_ok = __shfl_sync(kFull, free_ok, 0);
            if (!free_ok) {
                if (lane == 0) flag(c.dev_status, EKV_DEV_TIMEOUT);
                break;
            }
            mbar_try_wait(&bar_empty[buf], ph ^ 1);  // observe the release in every lane
            if (it >= items) {
                if (lane == 0) {
                    item_s[buf] = -1;
                    mbar_arrive(&bar_full[buf]);
                }
                break;
            }
            if (lane < a.CP) {
                blk_s[buf][lane] = blk;
                ntok_s[buf][lane] = nt;
            }
            const uint32_t bytes = (uint32_t)(nt * RB) * (SOFTMAX ? 2u : 1u);
            const uint32_t total = (uint32_t)warp_sum((int)bytes) + (uint32_t)(G * D * ESZ);
            if (lane == 0) item_s[buf] = it;
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&bar_full[buf], total);
            __syncwarp();
            unsigned char *st = stage0 + buf * stage_bytes;
            fence_proxy_async();
            if (lane == 0) {
                const int b = bh / H, h = bh % H;
                bulk_copy_g2s(st, qc + ((size_t)b * a.H_q + (size_t)h * G) * D * ESZ,
                              (uint32_t)(G * D * ESZ), &bar_full[buf]);
            }
            if (lane < a.CP && nt > 0) {
                const int h = bh % H;
                unsigned char *dst = st + QB + lane * P * RB;
                const size_t off = ((size_t)blk * H + h) * P * RB;
                bulk_copy_g2s(dst, kc + off, (uint32_t)(nt * RB), &bar_full[buf]);
                if (SOFTMAX) bulk_copy_g2s(dst + CT * RB, vc + off, (uint32_t)(nt * RB), &bar_full[buf]);
            }
            it += gridDim.x;
            advance();  // resolve the next item while this one's copies are in flight
        }
        pdl_trigger();
        return;
    }

    // ---------------------------------------------------------------------- consumers
    const int cidx = lane % W;
    for (int k = 0;; ++k) {
        const int buf = k % NS;
        const uint32_t ph = (k / NS) & 1;
        if (tid == 0) ok_s = (int)mbar_wait_bounded(&bar_full[buf], ph);
        named_sync(1, kNW * 32);
        if (!ok_s) {
            if (tid == 0) {
                flag(c.dev_status, EKV_DEV_TIMEOUT);
                mbar_wait_bounded(&bar_full[buf], ph);  // let any copy still in flight land
            }
            break;
        }
        mbar_try_wait(&bar_full[buf], ph);  // observe the completed phase in every thread
        const long long it = item_s[buf];
        if (it < 0) break;
        const int ci = (int)(it / BH), bh = (int)(it % BH);
        const int b = bh / H, h = bh % H;
        const unsigned char *st = stage0 + buf * stage_bytes;
        const unsigned char *tile = st + QB;
        const int *ntok = ntok_s[buf];

        float qv[G][EPC];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float f[EPC];
            Chunk<DT>::unpack(*reinterpret_cast<const uint4 *>(st + g * RB + cidx * 16), f);
#pragma unroll
            for (int e = 0; e < EPC; ++e) qv[g][e] = a.qscale * f[e];
        }

        // ---- logits of the chunk's tokens, from shared memory
        for (int base = warp * TW; base < CT; base += kNW * TW) {
            uint4 x[TPL];
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
                const int slot = base + i * RPI + lane / W;
                x[i] = *reinterpret_cast<const uint4 *>(tile + slot * RB + cidx * 16);
            }
            float part[NQK];
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
                float f[EPC];
                Chunk<DT>::unpack(x[i], f);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float s = 0.f;
#pragma unroll
                    for (int e = 0; e < EPC; ++e) s = fmaf(qv[g][e], f[e], s);
                    part[i * G + g] = s;
                }
            }
            transpose_reduce<NQK, W>(part, lane);
            if (NQK >= W || ((lane % W) % (W / NQK)) == 0) {
#pragma unroll
                for (int r = 0; r < OUTN; ++r) {
                    const int idx = transpose_index<NQK, W>(lane, r);
                    const int i = idx / G, g = idx % G;
                    const int slot = base + i * RPI + lane / W;
                    const int pi = slot >> a.Pshift, t = slot & (P - 1);
                    z_s[g * CT + slot] = t < ntok[pi] ? part[r] : -INFINITY;
                }
            }
        }
        named_sync(1, kNW * 32);
        if (warp < G) {
            float m = -INFINITY;
            for (int s = lane; s < CT; s += 32) m = fmaxf(m, z_s[warp * CT + s]);
            m = warp_max(m);
            if (lane == 0) m_s[warp] = m;
        }
        named_sync(1, kNW * 32);
        const size_t bq0 = (size_t)b * a.H_q + h * G;

        if constexpr (!SOFTMAX) {
            mbar_arrive(&bar_empty[buf]);  // the stage is no longer read
            for (int i = tid; i < G * CT; i += kNW * 32) {
                const int g = i / CT, s = i - g * CT;
                a.logits[(bq0 + g) * (size_t)a.LS + (size_t)ci * CT + s] = z_s[g * CT + s];
            }
            if (tid < G) a.part_ml[((bq0 + tid) * a.NC + ci) * 2] = m_s[tid];
            named_sync(1, kNW * 32);
            continue;
        } else {
            // ---- softmax partial: p = 2^(z - m), l = sum p, o = sum p v (V tile after K)
            for (int i = tid; i < G * CT; i += kNW * 32) {
                const int g = i / CT;
                const float z = z_s[i];
                z_s[i] = z == -INFINITY ? 0.f : exp2f(z - m_s[g]);
            }
            named_sync(1, kNW * 32);
            if (warp < G) {
                float l = 0.f;
                for (int s = lane; s < CT; s += 32) l += z_s[warp * CT + s];
                l = warp_sum(l);
                if (lane == 0) l_s[warp] = l;
            }
            float acc[G][EPC];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[g][e] = 0.f;
            const unsigned char *vt = tile + CT * RB;
            for (int base = warp * TW; base < CT; base += kNW * TW) {
                uint4 x[TPL];
#pragma unroll
                for (int i = 0; i < TPL; ++i) {
                    const int slot = base + i * RPI + lane / W;
                    x[i] = *reinterpret_cast<const uint4 *>(vt + slot * RB + cidx * 16);
                }
#pragma unroll
                for (int i = 0; i < TPL; ++i) {
                    const int slot = base + i * RPI + lane / W;
                    float f[EPC];
                    Chunk<DT>::unpack(x[i], f);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float p = z_s[g * CT + slot];
                        if (p != 0.f) {  // rows past a page's valid tokens hold stale data
#pragma unroll
                            for (int e = 0; e < EPC; ++e) acc[g][e] = fmaf(p, f[e], acc[g][e]);
                        }
                    }
                }
            }
            mbar_arrive(&bar_empty[buf]);  // the stage is no longer read
#pragma unroll
            for (int o = W; o < 32; o <<= 1)
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int e = 0; e < EPC; ++e) acc[g][e] += __shfl_xor_sync(kFull, acc[g][e], o);
            if (lane < W) {
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int e = 0; e < EPC; ++e) o_s[(warp * G + g) * D + cidx * EPC + e] = acc[g][e];
            }
            named_sync(1, kNW * 32);
            for (int i = tid; i < G * D; i += kNW * 32) {
                float s = 0.f;
#pragma unroll
                for (int w = 0; w < kNW; ++w) s += o_s[w * G * D + i];
                const int g = i / D, dd = i - g * D;
                a.part_o[((bq0 + g) * a.NC + ci) * D + dd] = s;
            }
            if (tid < G) {
                a.part_ml[((bq0 + tid) * a.NC + ci) * 2] = m_s[tid];
                a.part_ml[((bq0 + tid) * a.NC + ci) * 2 + 1] = l_s[tid];
            }
            named_sync(1, kNW * 32);
        }
    }
    pdl_trigger();
}

// ------------------------------------------------------------------------------ finish
template <int D>
__device__ void finish_softmax(const DecodeArgs &a, int b, int hq, int nchunks)
{
    __shared__ float red[kNW];
    __shared__ float o_acc[256];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t bq = (size_t)b * a.H_q + hq;
    const float *ml = a.part_ml + bq * a.NC * 2;
    float M = -INFINITY;
    for (int ch = tid; ch < nchunks; ch += 256) M = fmaxf(M, __ldcg(ml + 2 * ch));
    M = warp_max(M);
    if (lane == 0) red[warp] = M;
    __syncthreads();
    M = red[0];
#pragma unroll
    for (int w = 1; w < kNW; ++w) M = fmaxf(M, red[w]);
    __syncthreads();
    float L = 0.f;
    for (int ch = tid; ch < nchunks; ch += 256) {
        const float m = __ldcg(ml + 2 * ch);
        if (m != -INFINITY) L += exp2f(m - M) * __ldcg(ml + 2 * ch + 1);
    }
    L = warp_sum(L);
    if (lane == 0) red[warp] = L;
    __syncthreads();
    L = 0.f;
#pragma unroll
    for (int w = 0; w < kNW; ++w) L += red[w];
    constexpr int SPLIT = 256 / D;
    const int dd = tid % D, part = tid / D;
    float acc = 0.f;
    if (M != -INFINITY) {
#pragma unroll 8
        for (int ch = part; ch < nchunks; ch += SPLIT) {
            const float m = __ldcg(ml + 2 * ch);
            if (m != -INFINITY)
                acc = fmaf(exp2f(m - M), __ldcg(a.part_o + (bq * a.NC + ch) * D + dd), acc);
        }
    }
    o_acc[tid] = acc;
    __syncthreads();
    if (tid < D) {
        float s = 0.f;
#pragma unroll
        for (int p2 = 0; p2 < SPLIT; ++p2) s += o_acc[p2 * D + tid];
        a.out[bq * D + tid] = M == -INFINITY ? 0.f : s / L;
    }
    if (tid == 0) a.stat[bq] = M == -INFINITY ? -INFINITY : (M + log2f(L)) * 0.69314718055994530942f;
}

constexpr int kCapW = 512;       // gathered logits per warp kept in shared memory
constexpr int kHistBins = 512;   // bins per level of the threshold bracket (two per thread)
constexpr int kHistLevels = 4;   // bracket levels before the tie fallback
constexpr int kHistExact = 128;  // a bracket range with at most this many logits is solved exactly
constexpr int kActCap = 1024;    // active chunks listed by the finish (more: walk every chunk)

// Exact threshold over a known part of the support -- n0 logits with sums a0 = sum x,
// b0 = sum x^2, every one above all candidates -- plus at most 32*R candidates held R per lane
// as y = x - lo >= 0 (-inf padding). Same rule as warp_exact_tau on the merged sorted order: the
// support is the largest k with tau(k) <= x_(k); if no candidate qualifies it is the known part.
template <int R>
__device__ double warp_exact_tau_based(float (&y)[R], int cnt, double lo, double n0, double a0,
                                       double b0, bool sparsemax)
{
    const int lane = threadIdx.x & 31;
    warp_sort_desc<R>(y);
    int bk = 0;  // candidates in the support (0: the known part alone)
    double bx = 0.0, bxx = 0.0;
    float carry1 = 0.f, carry2 = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = r * 32 + lane;
        const bool in = e < cnt;
        const float yd = in ? y[r] : 0.f;
        float s1 = yd, s2 = yd * yd;  // small: y lies within one bracket bin
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float t1 = __shfl_up_sync(kFull, s1, o), t2 = __shfl_up_sync(kFull, s2, o);
            if (lane >= o) { s1 += t1; s2 += t2; }
        }
        s1 += carry1;
        s2 += carry2;
        carry1 = __shfl_sync(kFull, s1, 31);
        carry2 = __shfl_sync(kFull, s2, 31);
        const double k = (double)(e + 1);
        const double sx = k * lo + (double)s1;
        const double sxx = k * lo * lo + 2.0 * lo * (double)s1 + (double)s2;
        const bool ok = in && closed_form_ok(n0 + k, a0 + sx, b0 + sxx, lo + (double)yd, sparsemax);
        const unsigned bal = __ballot_sync(kFull, ok);
        if (bal) {  // later rows win
            const int src = 31 - __clz(bal);
            bk = r * 32 + src + 1;
            bx = __shfl_sync(kFull, sx, src);
            bxx = __shfl_sync(kFull, sxx, src);
        }
    }
    if (n0 + bk == 0.0) return lo;
    double tau = lo;
    closed_form_tau(n0 + bk, a0 + bx, b0 + bxx, sparsemax, tau);
    return tau;
}

// Block-wide suffix sums (inclusive, from the highest thread down) of three doubles.
__device__ __forceinline__ void block_suffix3(double (&v)[3], double (*wtot)[3])
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const double t = __shfl_down_sync(kFull, v[i], o);
            if (lane + o < 32) v[i] += t;
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 3; ++i) wtot[warp][i] = v[i];
    }
    __syncthreads();
    for (int w = warp + 1; w < kNW; ++w) {
#pragma unroll
        for (int i = 0; i < 3; ++i) v[i] += wtot[w][i];
    }
}

struct HistScratch {
    int c[kHistBins];        // logits per bin of the current range
    double base[3];          // count, sum x, sum x^2 of the logits above the current range
    double wtot[kNW][3];
    float list[kHistExact];
    int nlist;
    int jlo, jhi;
};

// The threshold bracket, in the domain x = z - zmax (candidates in (-1, 0]). F(t) = sum
// (x - t)_+^p (p = 2 for 1.5-entmax, 1 for sparsemax) is decreasing and tau solves F(tau) = 1
// with tau >= -1. A level counts the candidates of its range [lo, hi) in bins of a power-of-two
// width (exact binning in fp64). With only counts, F at a bin edge e is bracketed by placing
// every logit at its bin's lower or upper edge: F_lo(e) <= F(e) <= F_hi(e). The last edge with
// F_lo >= 1 is a lower bound on tau, the first edge after it with F_hi < 1 an upper bound; the
// logits above the upper bound are in the support and join the known part `base` (exact sums),
// those below the lower bound are out, and the bins between form the next range. The top
// level's range is (-1, 0] (its last bin also takes x = 0); a range that reaches the top of a
// closed range stays closed, so the maximum never drops out.
struct HistRange {
    double lo, hi, bw, inv;
    int nb;     // bins in use
    bool top;   // closed at hi
    __device__ void set(double lo_, double hi_, double bw_, bool top_)
    {
        lo = lo_; hi = hi_; bw = bw_; inv = 1.0 / bw_; top = top_;
        nb = (int)ceil((hi - lo) * inv);
        nb = nb < 1 ? 1 : (nb > kHistBins ? kHistBins : nb);
    }
    __device__ __forceinline__ int bin(double xd) const
    {
        if (xd < lo || (!top && xd >= hi)) return -1;
        const int k = (int)((xd - lo) * inv);
        return k < nb - 1 ? k : nb - 1;
    }
};

__device__ __forceinline__ void hist_count(HistScratch &H, const HistRange &R, double xd)
{
    const int k = R.bin(xd);
    if (k >= 0) atomicAdd(&H.c[k], 1);
}

// Zero the bins (block-wide; a __syncthreads must follow before the first hist_count).
__device__ __forceinline__ void hist_clear(HistScratch &H, bool reset_base)
{
    for (int i = threadIdx.x; i < kHistBins; i += 256) H.c[i] = 0;
    if (threadIdx.x == 0) {
        H.jlo = 0;
        H.jhi = 0;
        H.nlist = 0;
        if (reset_base) H.base[0] = H.base[1] = H.base[2] = 0.0;
    }
}

// Block-wide sum of three doubles per thread (every thread gets the total).
__device__ __forceinline__ void block_sum3(double (&v)[3], double (*wtot)[3])
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < 3; ++i) v[i] = warp_sum(v[i]);
    __syncthreads();
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 3; ++i) wtot[warp][i] = v[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < kNW; ++w) s += wtot[w][i];
        v[i] = s;
    }
    __syncthreads();
}

// With the bins of range R counted: the bracketing bins [jlo, jhi) into H.jlo, H.jhi. Every
// thread of the block must call this.
__device__ void hist_bracket(HistScratch &H, const HistRange &R, bool sparsemax)
{
    const int tid = threadIdx.x;
    __syncthreads();
    // suffix sums from bin 2*tid of (count, count*k, count*k^2)
    double own[2][3], suf[3];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int k = 2 * tid + r;
        const double cc = k < R.nb ? (double)H.c[k] : 0.0;
        own[r][0] = cc;
        own[r][1] = cc * k;
        own[r][2] = cc * k * k;
    }
#pragma unroll
    for (int i = 0; i < 3; ++i) suf[i] = own[0][i] + own[1][i];
    block_suffix3(suf, H.wtot);
    const double n0 = H.base[0], a0 = H.base[1], b0 = H.base[2], bw = R.bw;
    // F at edge j with every logit of bin k >= j placed at edge k + off (off = 0 or 1)
    auto F_edge = [&](int j, const double (&s)[3], int off) {
        const double e = R.lo + j * bw;
        const double C = s[0], K1 = s[1] + off * s[0], K2 = s[2] + 2.0 * off * s[1] + off * s[0];
        if (sparsemax) return (a0 - e * n0) + bw * (K1 - j * C);
        return (b0 - 2.0 * e * a0 + e * e * n0) + bw * bw * (K2 - 2.0 * j * K1 + (double)j * j * C);
    };
    double suf1[3];  // suffix from bin 2*tid+1
#pragma unroll
    for (int i = 0; i < 3; ++i) suf1[i] = suf[i] - own[0][i];
    const int j0 = 2 * tid, j1 = 2 * tid + 1;
    int lo_m = -1, hi_m = -1;
    if (j1 < R.nb && F_edge(j1, suf1, 0) >= 1.0) lo_m = j1;
    else if (j0 < R.nb && F_edge(j0, suf, 0) >= 1.0) lo_m = j0;
    if (j1 < R.nb && F_edge(j1, suf1, 1) >= 1.0) hi_m = j1;
    else if (j0 < R.nb && F_edge(j0, suf, 1) >= 1.0) hi_m = j0;
    if (lo_m >= 0) atomicMax(&H.jlo, lo_m);
    if (hi_m >= 0) atomicMax(&H.jhi, hi_m + 1);
    __syncthreads();
    const int jlo = H.jlo, jhi = max(H.jhi, jlo + 1);
    __syncthreads();
    if (tid == 0) H.jhi = jhi;
    __syncthreads();
}

// Add the logits of range R at and above bin jhi to H.base (exact fp64 sums). `visit(fn)` calls
// fn(x) for every candidate of the calling warp; every thread of the block must call this.
template <typename Visit>
__device__ void hist_add_base(Visit &&visit, HistScratch &H, const HistRange &R, int jhi)
{
    double acc[3] = {0.0, 0.0, 0.0};
    if (jhi < R.nb) {
        visit([&](float x) {
            const double xd = x;
            if (R.bin(xd) >= jhi) { acc[0] += 1.0; acc[1] += xd; acc[2] += xd * xd; }
        });
    }
    block_sum3(acc, H.wtot);
    if (threadIdx.x == 0) {
        H.base[0] += acc[0];
        H.base[1] += acc[1];
        H.base[2] += acc[2];
    }
    __syncthreads();
}

// tau once range R (its logits counted in H.c) brackets it: with at most kHistExact logits in
// the range one warp solves exactly over them plus the known part; with more (ties to within
// the last level's bin width) the range is taken whole or not at all. Every thread of the
// block must call this.
template <typename Visit>
__device__ double hist_solve(Visit &&visit, HistScratch &H, const HistRange &R, int cnt_range,
                             bool sparsemax)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const double flo = R.lo;
    const double N0 = H.base[0], A0 = H.base[1], B0 = H.base[2];
    if (cnt_range <= kHistExact) {
        if (threadIdx.x == 0) H.nlist = 0;
        __syncthreads();
        visit([&](float x) {
            const double xd = x;
            if (R.bin(xd) < 0) return;
            const int pos = atomicAdd(&H.nlist, 1);
            if (pos < kHistExact) H.list[pos] = (float)(xd - flo);
        });
        __syncthreads();
        if (warp == 0) {
            const int n = H.nlist < kHistExact ? H.nlist : kHistExact;
            float y[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int e = r * 32 + lane;
                y[r] = e < n ? H.list[e] : -INFINITY;
            }
            double tau;
            if (n <= 32) {
                float y1[1] = {y[0]};
                tau = warp_exact_tau_based<1>(y1, n, flo, N0, A0, B0, sparsemax);
            } else if (n <= 64) {
                float y2[2] = {y[0], y[1]};
                tau = warp_exact_tau_based<2>(y2, n, flo, N0, A0, B0, sparsemax);
            } else {
                tau = warp_exact_tau_based<4>(y, n, flo, N0, A0, B0, sparsemax);
            }
            if (lane == 0) H.wtot[0][0] = tau;
        }
        __syncthreads();
        const double tau = H.wtot[0][0];
        __syncthreads();
        return tau;
    }
    // more than kHistExact logits within the last level's bin width: ties at the resolution of
    // the logits. Equal logits are in the support together or not at all, so the range joins
    // the support as a block if the closed form over the known part plus the whole range falls
    // below the range, and stays out otherwise.
    double acc[3] = {0.0, 0.0, 0.0};
    double rmin = INFINITY;
    visit([&](float x) {
        const double xd = x;
        if (R.bin(xd) >= 0) { acc[0] += 1.0; acc[1] += xd; acc[2] += xd * xd; rmin = fmin(rmin, xd); }
    });
    rmin = -warp_max((float)-rmin);
    block_sum3(acc, H.wtot);
    if (lane == 0) H.list[warp] = (float)rmin;
    __syncthreads();
    float lo_r = H.list[0];
#pragma unroll
    for (int w = 1; w < kNW; ++w) lo_r = fminf(lo_r, H.list[w]);
    __syncthreads();
    double tau = flo;
    if (closed_form_tau(N0 + acc[0], A0 + acc[1], B0 + acc[2], sparsemax, tau) && tau < (double)lo_r)
        return tau;
    tau = flo;
    if (N0 > 0.0) closed_form_tau(N0, A0, B0, sparsemax, tau);
    return tau;
}

template <int DT, int D>
__device__ void finish_entmax_cta(const DecodeArgs &a, int b, int h, int hq, int nsel, int nchunks)
{
    constexpr int EPC = Chunk<DT>::N;
    constexpr int ESZ = Chunk<DT>::kBytes;
    constexpr int W = D * ESZ / 16;
    constexpr int RPI = 32 / W;
    constexpr int UNRV = 8;  // V rows in flight per lane group
    constexpr int UNR = 4;   // float4 logit loads in flight per lane while gathering
    __shared__ float cz[kNW][kCapW];
    __shared__ int cs[kNW][kCapW];
    __shared__ int cn[kNW];
    __shared__ float red[kNW];
    __shared__ double s_tau;
    __shared__ float o_w[kNW][D];
    __shared__ HistScratch hist;
    __shared__ int act[kActCap];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const ekv_cache &c = a.c;
    const int P = c.page_size, H = c.num_kv_heads;
    const size_t bq = (size_t)b * a.H_q + hq;
    const float *z = a.logits + bq * (size_t)a.LS;
    const bool sparsemax = a.alpha == 2.0f;

    hist_clear(hist, true);
    const float *ml = a.part_ml + bq * a.NC * 2;
    float zmax = -INFINITY, mv[4];  // chunk maxima; the first 1024 stay in registers
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int ch = tid + 256 * r;
        mv[r] = ch < nchunks ? __ldcg(ml + 2 * ch) : -INFINITY;
        zmax = fmaxf(zmax, mv[r]);
    }
    for (int ch = tid + 1024; ch < nchunks; ch += 256) zmax = fmaxf(zmax, __ldcg(ml + 2 * ch));
    zmax = warp_max(zmax);
    if (lane == 0) red[warp] = zmax;
    __syncthreads();
    zmax = red[0];
#pragma unroll
    for (int w = 1; w < kNW; ++w) zmax = fmaxf(zmax, red[w]);
    if (zmax == -INFINITY) {  // no valid token among the selected pages
        for (int i = tid; i < D; i += 256) a.out[bq * D + i] = 0.f;
        if (tid == 0) a.stat[bq] = -INFINITY;
        return;
    }
    const float thr = zmax - 1.0f;  // the largest weight is at most 1, so tau >= zmax - 1

    // A lower bound on tau from the chunk maxima: they are logits, and the exact threshold of
    // any subset of the logits is at most that of all of them. Each warp solves exactly over the
    // maxima it holds (32, or 128 when there are more than 256 chunks); no logit at or below the
    // largest bound can carry weight. Candidates are z > thr with x = z - zmax >= clo.
    double clo = -INFINITY;
    {
        float lbw = -INFINITY;
        if (nchunks <= 256) {
            float v1[1] = {mv[0] - zmax};
            const int nv = __popc(__ballot_sync(kFull, mv[0] > thr));
            if (nv > 1) lbw = (float)warp_exact_tau<1>(v1, nv, sparsemax);
        } else {
            float v4[4];
            int nv = 0;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                v4[r] = mv[r] - zmax;
                nv += __popc(__ballot_sync(kFull, mv[r] > thr));
            }
            if (nv > 1) lbw = (float)warp_exact_tau<4>(v4, nv, sparsemax);
        }
        __syncthreads();  // every warp has read zmax from red[]
        if (lane == 0) red[warp] = lbw;
        __syncthreads();
        float lb = red[0];
#pragma unroll
        for (int w = 1; w < kNW; ++w) lb = fmaxf(lb, red[w]);
        // lowered a little so that the fp32 rounding of the bound never drops a support member
        clo = (double)lb - 1e-6 * fmax(1.0, fabs((double)lb));
        __syncthreads();
    }

    // active chunks: those whose maximum is a candidate (no other chunk holds one), listed in
    // order; with more than kActCap of them every chunk is walked
    int nact = 0;
    for (int ch0 = 0; ch0 < nchunks; ch0 += 256) {
        const int ch = ch0 + tid;
        const int r = ch0 >> 8;
        const float m = r == 0 ? mv[0] : (r == 1 ? mv[1] : (r == 2 ? mv[2] : (r == 3 ? mv[3]
                      : (ch < nchunks ? __ldcg(ml + 2 * ch) : -INFINITY))));
        const int keep = m > thr && (double)(m - zmax) >= clo;
        int tot;
        const int pos = nact + block_incl_scan<256>(keep, cn, &tot) - keep;
        if (keep && pos < kActCap) act[pos] = ch;
        nact += tot;
    }
    const bool dense = nact > kActCap;
    if (dense) nact = nchunks;
    __syncthreads();

    // gather: the active chunks form a virtual run of nact * CT slots; warp w owns a contiguous
    // range of its float4 groups [f0w, f1w). Candidates (x = z - zmax and the slot) are listed,
    // the first kCapW of each warp
    const int CT = a.CP * P, CT4 = CT / 4;
    const int nf4 = nact * CT4;
    const int perf = (nf4 + kNW - 1) / kNW;
    const int f0w = min(warp * perf, nf4), f1w = min(f0w + perf, nf4);
    auto slot_of = [&](int f) {  // first slot of virtual float4 group f
        const int i = f / CT4;
        return (dense ? i : act[i]) * CT + (f - i * CT4) * 4;
    };
    // (clo rises again once the top level of the threshold bracket is bracketed)
    auto gather = [&]() {
        int cnt = 0;
        for (int f = f0w; f < f1w; f += 32 * UNR) {
            float4 v[UNR];
            int sl[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int fu = f + u * 32 + lane;
                sl[u] = fu < f1w ? slot_of(fu) : 0;
                v[u] = fu < f1w ? __ldcg(reinterpret_cast<const float4 *>(z + sl[u]))
                                : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const float e4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x = e4[e] - zmax;
                    const bool keep = e4[e] > thr && (double)x >= clo;
                    const unsigned bal = __ballot_sync(kFull, keep);
                    const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
                    if (keep && pos < kCapW) {
                        cz[warp][pos] = x;
                        cs[warp][pos] = sl[u] + e;
                    }
                    cnt += __popc(bal);
                }
            }
        }
        return cnt;
    };
    int cnt = gather();
    __syncthreads();
    if (lane == 0) cn[warp] = cnt;
    __syncthreads();
    bool any_over = false;
    int total = 0;
#pragma unroll
    for (int w = 0; w < kNW; ++w) {
        any_over |= cn[w] > kCapW;
        total += cn[w];
    }
    bool over = cnt > kCapW;
    // this warp's candidates: its list, or its range of the active chunks again when the list
    // overflowed
    auto visit_own = [&](auto &&fn) {
        if (!over) {
            for (int i = lane; i < cnt; i += 32) fn(cz[warp][i]);
        } else {
            for (int i = lane; i < (f1w - f0w) * 4; i += 32) {
                const float v = __ldcg(z + slot_of(f0w + i / 4) + (i & 3));
                const float x = v - zmax;
                if (v > thr && (double)x >= clo) fn(x);
            }
        }
    };
    // Resolve the listed candidates' cache rows now (the chunk kernel recorded each selected
    // page's block) and start their V rows towards L2: the support is among them, so its rows
    // are on their way while tau is solved. A list refilled later holds slots again.
    const char *vc = static_cast<const char *>(c.v_cache);
    const int32_t *blk_row = a.sel_blk + ((size_t)b * H + h) * a.max_sel;
    bool rows_listed = false;
    if (!over) {
        for (int i = lane; i < cnt; i += 32) {
            const int slot = cs[warp][i], t = slot & (P - 1);
            const int blk = __ldcg(blk_row + (slot >> a.Pshift));
            cs[warp][i] = blk * P + t;
            const char *vrow = vc + (((size_t)blk * H + h) * P + t) * D * ESZ;
#pragma unroll
            for (int off = 0; off < D * ESZ; off += 128) prefetch_l2(vrow + off);
        }
        rows_listed = true;
    }
    HistRange R;
    R.set(-1.0, 0.0, 1.0 / kHistBins, true);

    double tau;  // in the shifted domain x = z - zmax
    if (!any_over && total <= 128) {
        // one warp sorts every candidate (no block barrier on this path): element e = r * 32 +
        // lane is the e-th in warp order
        if (warp == 0) {
            auto load = [&](int e) {
                int base = 0;
                float x = -INFINITY;
#pragma unroll
                for (int w = 0; w < kNW; ++w) {
                    if (e >= base && e < base + cn[w]) x = cz[w][e - base];
                    base += cn[w];
                }
                return x;
            };
            double t;
            if (total <= 32) {
                float x1[1] = {load(lane)};
                t = warp_exact_tau<1>(x1, total, sparsemax);
            } else if (total <= 64) {
                float x2[2] = {load(lane), load(32 + lane)};
                t = warp_exact_tau<2>(x2, total, sparsemax);
            } else {
                float x4[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) x4[r] = load(r * 32 + lane);
                t = warp_exact_tau<4>(x4, total, sparsemax);
            }
            if (lane == 0) s_tau = t;
        }
        __syncthreads();
        tau = s_tau;
    } else {
        visit_own([&](float x) { hist_count(hist, R, (double)x); });
        for (int level = 0;; ++level) {
            hist_bracket(hist, R, sparsemax);
            const int jlo = hist.jlo, jhi = hist.jhi;
            int cr = 0;
            for (int k = jlo; k < jhi; ++k) cr += hist.c[k];
            const double nlo = R.lo + jlo * R.bw, nhi = R.lo + jhi * R.bw;
            const bool ntop = R.top && jhi >= R.nb;
            // bins of the next range: the power-of-two width that covers it in kHistBins
            double nbw = R.bw;
            while (nbw * kHistBins > (jhi - jlo) * R.bw * 2.0 && nbw > 0x1p-60) nbw *= 0.5;
            if (level == 0 && any_over) {
                // only logits at or above the lower bound can be in the support: an overflowed
                // warp lists those again
                clo = nlo;
                if (over) {
                    cnt = gather();
                    over = cnt > kCapW;
                    rows_listed = false;  // the new list holds slots
                }
            }
            hist_add_base(visit_own, hist, R, jhi);
            R.set(nlo, nhi, nbw, ntop);
            if (cr <= kHistExact || level == kHistLevels - 1) {
                tau = hist_solve(visit_own, hist, R, cr, sparsemax);
                break;
            }
            hist_clear(hist, false);
            __syncthreads();
            visit_own([&](float x) { hist_count(hist, R, (double)x); });
        }
    }

    // o = sum over the support of p_i v_i, each warp over its own entries: compact the support
    // (weight, row) in place over the gathered list -- rows resolved above, or slots resolved
    // here with all lookups in flight -- then stream the V rows UNRV per lane group; a warp whose
    // list overflowed does this in rounds of at most kCapW entries
    const int cidx = lane % W, row = lane / W;
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
    float *sp = cz[warp];  // compacted support weights
    int *sr = cs[warp];    // and slots, then rows as blk * P + t
    const int nitems = over ? (f1w - f0w) * 4 : cnt;
    int it0 = 0;
    do {
        int ns = 0;
        while (it0 < nitems && ns <= kCapW - 32) {
            const int i = it0 + lane;
            float x = -INFINITY;
            int slot = 0;
            if (i < nitems) {
                if (over) {
                    slot = slot_of(f0w + i / 4) + (i & 3);
                    const float v = __ldcg(z + slot);
                    x = v > thr ? v - zmax : -INFINITY;
                } else {
                    slot = cs[warp][i];
                    x = cz[warp][i];
                }
            }
            const double r = (double)x - tau;
            const bool keep = r > 0.0;
            const unsigned bal = __ballot_sync(kFull, keep);
            __syncwarp();
            if (keep) {
                const int pos = ns + __popc(bal & ((1u << lane) - 1u));
                sp[pos] = (float)(sparsemax ? r : r * r);
                sr[pos] = slot;
            }
            __syncwarp();
            ns += __popc(bal);
            it0 += 32;
        }
        for (int k0 = rows_listed ? ns : 0; k0 < ns; k0 += 128) {
            int sl[4], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int k = k0 + u * 32 + lane;
                sl[u] = k < ns ? sr[k] : 0;
                bv[u] = k < ns ? __ldcg(blk_row + (sl[u] >> a.Pshift)) : 0;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int k = k0 + u * 32 + lane;
                if (k < ns) sr[k] = bv[u] * P + (sl[u] & (P - 1));
            }
        }
        __syncwarp();
        for (int k0 = 0; k0 < ns; k0 += RPI * UNRV) {
            uint4 xv[UNRV];
            float p[UNRV];
#pragma unroll
            for (int u = 0; u < UNRV; ++u) {
                const int k = k0 + u * RPI + row;
                p[u] = 0.f;
                xv[u] = make_uint4(0, 0, 0, 0);
                if (k < ns) {
                    p[u] = sp[k];
                    const int br = sr[k];
                    const size_t rowi = ((size_t)(br >> a.Pshift) * H + h) * P + (br & (P - 1));
                    xv[u] = ld_stream16(vc + rowi * D * ESZ + cidx * 16);
                }
            }
#pragma unroll
            for (int u = 0; u < UNRV; ++u) {
                float f[EPC];
                Chunk<DT>::unpack(xv[u], f);
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[e] = fmaf(p[u], f[e], acc[e]);
            }
        }
        __syncwarp();
    } while (it0 < nitems);
#pragma unroll
    for (int o = W; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[e] += __shfl_xor_sync(kFull, acc[e], o);
    if (lane < W) {
#pragma unroll
        for (int e = 0; e < EPC; ++e) o_w[warp][cidx * EPC + e] = acc[e];
    }
    __syncthreads();
    for (int i = tid; i < D; i += 256) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kNW; ++w) sum += o_w[w][i];
        a.out[bq * D + i] = sum;
    }
    if (tid == 0) a.stat[bq] = (float)(tau + (double)zmax);
}

template <int DT, int D, int G, bool SOFTMAX>
__global__ void __launch_bounds__(256, 3)
decode_finish_kernel(DecodeArgs a)
{
    // one CTA per (sequence, query head)
    pdl_wait();
    const int hq = blockIdx.x, b = blockIdx.y;
    const int h = hq / G, bh = b * a.c.num_kv_heads + h;
    int nsel = a.sel_count[bh];
    nsel = nsel < 0 ? 0 : (nsel > a.max_sel ? a.max_sel : nsel);
    const int nchunks = (nsel + a.CP - 1) / a.CP;
    const size_t bq = (size_t)b * a.H_q + hq;
    if (nchunks == 0) {
        for (int i = threadIdx.x; i < D; i += 256) a.out[bq * D + i] = 0.f;
        if (threadIdx.x == 0) a.stat[bq] = -INFINITY;
    } else if constexpr (SOFTMAX) {
        finish_softmax<D>(a, b, hq, nchunks);
    } else {
        finish_entmax_cta<DT, D>(a, b, h, hq, nsel, nchunks);
    }
    pdl_trigger();
}

// ------------------------------------------------------------------------------ host side
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace layout of one attention mode: [B*H_q][NC][2] chunk (m, l) | [B*H_q][NC][D] chunk
// sums (softmax) | [B*H_q][NC*CP*P] logits (entmax) | [B*H_kv][max_sel] cache block of every
// selected page (entmax), each 256-byte aligned.
static size_t mode_layout(int batch, int H_q, int H, int D, int P, int dtype, int max_sel,
                          bool softmax, size_t *off_o, size_t *off_logits, size_t *off_blk,
                          int *CP, int *NC)
{
    const int rb = D * (dtype == EKV_BF16 ? 2 : 4);
    // bf16 chunks served by the tensor-core kernels are one 128-token tile (entmax; softmax at
    // d = 128)
    const bool tc = dtype == EKV_BF16 && (!softmax || D == 128);
    const int cp = tc ? 128 / P : chunk_tokens(rb, P, softmax) / P;
    const int nc = (max_sel + cp - 1) / cp;
    const size_t BQ = (size_t)batch * H_q;
    size_t off = align256(BQ * nc * 2 * sizeof(float));
    if (off_o) *off_o = off;
    off += align256(BQ * nc * D * sizeof(float));
    if (off_logits) *off_logits = off;
    off += align256(BQ * (size_t)nc * cp * P * sizeof(float));
    if (off_blk) *off_blk = off;
    off += align256((size_t)batch * H * max_sel * sizeof(int32_t));
    if (CP) *CP = cp;
    if (NC) *NC = nc;
    return off;
}

// Bytes that cover every attention mode.
size_t decode_workspace_bytes_all_modes(int batch, int H_q, int H, int D, int P, int dtype,
                                        int max_sel)
{
    const size_t a = mode_layout(batch, H_q, H, D, P, dtype, max_sel, true, nullptr, nullptr,
                                 nullptr, nullptr, nullptr);
    const size_t b = mode_layout(batch, H_q, H, D, P, dtype, max_sel, false, nullptr, nullptr,
                                 nullptr, nullptr, nullptr);
    return a > b ? a : b;
}

template <int DT, int D, int G, bool SOFTMAX>
static cudaError_t launch_chunk(const DecodeArgs &a, cudaLaunchConfig_t cfg)
{
    constexpr int RB = D * Chunk<DT>::kBytes;
    auto k = decode_chunk_kernel<DT, D, G, SOFTMAX>;
    const int CT = a.CP * a.c.page_size;
    const size_t stage = (size_t)stage_q_bytes(G, D, Chunk<DT>::kBytes) + (size_t)CT * RB * (SOFTMAX ? 2 : 1);
    const size_t fixed = sizeof(float) * G * CT + (SOFTMAX ? sizeof(float) * kNW * G * D : 0);
    DecodeArgs a2 = a;
    a2.stages = kStages * stage + fixed <= 220 * 1024 ? kStages : 2;
    const size_t smem = a2.stages * stage + fixed;
    static bool attr_set = false;  // per instantiation
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    const long long items = (long long)a.c.batch * a.c.num_kv_heads * a.NC;
    const long long grid = persistent_grid_size((const void *)k, kThreads, smem);
    cfg.gridDim = dim3((unsigned)(items < grid ? items : grid));
    return cudaLaunchKernelEx(&cfg, k, a2);
}

bool tc_chunk_supported(const ekv_cache &c, int H_q, bool softmax);
cudaError_t launch_chunk_tc(const DecodeArgs &a, int G, cudaLaunchConfig_t cfg);
cudaError_t launch_softmax_tc(const DecodeArgs &a, int G, cudaLaunchConfig_t cfg);
bool direct_logits_supported(const ekv_cache &c, int H_q);
cudaError_t launch_logits_direct(const DecodeArgs &a, int G, cudaLaunchConfig_t cfg, bool *launched);

template <int DT, int D, int G>
static cudaError_t launch_decode_t(const DecodeArgs &a, bool softmax, cudaStream_t st, bool pdl)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e = cudaSuccess;
    const bool tc = DT == EKV_BF16 && tc_chunk_supported(a.c, a.H_q, softmax);
    bool direct = false;
    if (!softmax && tc && direct_logits_supported(a.c, a.H_q)) e = launch_logits_direct(a, G, cfg, &direct);
    if (e != cudaSuccess) return e;
    if (softmax)
        e = tc ? launch_softmax_tc(a, G, cfg) : launch_chunk<DT, D, G, true>(a, cfg);
    else if (!direct)
        e = tc ? launch_chunk_tc(a, G, cfg) : launch_chunk<DT, D, G, false>(a, cfg);
    if (e != cudaSuccess) return e;
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.gridDim = dim3(a.H_q, a.c.batch);
    cfg.numAttrs = 1;  // the finish kernel always waits on the chunk kernel programmatically
    if (softmax) return cudaLaunchKernelEx(&cfg, decode_finish_kernel<DT, D, G, true>, a);
    return cudaLaunchKernelEx(&cfg, decode_finish_kernel<DT, D, G, false>, a);
}

template <int DT, int D>
static cudaError_t launch_decode_g(const DecodeArgs &a, int G, bool softmax, cudaStream_t st, bool pdl)
{
    switch (G) {
    case 1: return launch_decode_t<DT, D, 1>(a, softmax, st, pdl);
    case 2: return launch_decode_t<DT, D, 2>(a, softmax, st, pdl);
    case 4: return launch_decode_t<DT, D, 4>(a, softmax, st, pdl);
    default: return launch_decode_t<DT, D, 8>(a, softmax, st, pdl);
    }
}


cudaError_t launch_sparse_decode(const ekv_cache &c, const void *q, int H_q, float scale,
                                 int attn, const int32_t *sel_idx, const int32_t *sel_count,
                                 int max_sel, float *out, float *stat, void *ws, cudaStream_t st,
                                 bool pdl)
{
    DecodeArgs a;
    size_t off_o, off_logits, off_blk;
    mode_layout(c.batch, H_q, c.num_kv_heads, c.head_dim, c.page_size, c.dtype, max_sel,
                attn == EKV_SOFTMAX, &off_o, &off_logits, &off_blk, &a.CP, &a.NC);
    a.LS = a.NC * a.CP * c.page_size;
    a.Pshift = c.page_size == 16 ? 4 : (c.page_size == 32 ? 5 : 6);
    a.c = c;
    a.q = q;
    a.H_q = H_q;
    a.alpha = attn == EKV_SOFTMAX ? 1.0f : (attn == EKV_ENTMAX15 ? 1.5f : 2.0f);
    a.qscale = attn == EKV_SOFTMAX ? scale * 1.44269504088896340736f : scale * (a.alpha - 1.0f);
    a.sel_idx = sel_idx;
    a.sel_count = sel_count;
    a.max_sel = max_sel;
    a.part_ml = static_cast<float *>(ws);
    a.part_o = reinterpret_cast<float *>(static_cast<char *>(ws) + off_o);
    a.logits = reinterpret_cast<float *>(static_cast<char *>(ws) + off_logits);
    a.sel_blk = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + off_blk);
    a.out = out;
    a.stat = stat;
    const bool softmax = attn == EKV_SOFTMAX;
    const int G = H_q / c.num_kv_heads;
    if (c.dtype == EKV_BF16)
        return c.head_dim == 128 ? launch_decode_g<EKV_BF16, 128>(a, G, softmax, st, pdl)
                                 : launch_decode_g<EKV_BF16, 64>(a, G, softmax, st, pdl);
    return c.head_dim == 128 ? launch_decode_g<EKV_F32, 128>(a, G, softmax, st, pdl)
                             : launch_decode_g<EKV_F32, 64>(a, G, softmax, st, pdl);
}

}  // namespace ekv
