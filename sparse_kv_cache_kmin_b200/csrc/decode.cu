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
#include "ekv_device.cuh"

namespace ekv {

struct DecodeArgs {
    ekv_cache c;
    const void *q;
    int H_q;
    float qscale;  // softmax: scale * log2(e); entmax: scale * (alpha - 1)
    float alpha;
    const int32_t *sel_idx;
    const int32_t *sel_count;
    int max_sel;
    int CP;         // pages per chunk
    int NC;         // chunks per (sequence, KV head) at most
    int LS;         // logits row stride: NC * CP * P
    int Pshift;     // log2(P)
    float *part_ml; // [B * H_q][NC][2]   softmax (m, l); entmax (max z, unused)
    float *part_o;  // [B * H_q][NC][D]   softmax sum p v
    float *logits;  // [B * H_q][LS]       entmax z
    float *out;
    float *stat;
};

constexpr int kChunkTok = 256;  // tokens per chunk at most
constexpr int kNW = 8;          // warps per CTA

template <int DT, int D, int G, bool SOFTMAX>
__global__ void __launch_bounds__(256)
decode_chunk_kernel(DecodeArgs a)
{
    constexpr int EPC = Chunk<DT>::N;
    constexpr int ESZ = Chunk<DT>::kBytes;
    constexpr int W = D * ESZ / 16;  // lanes per token row
    constexpr int RPI = 32 / W;      // rows per warp instruction
    constexpr int TPL = 4;           // rows per lane per step
    constexpr int TW = TPL * RPI;    // rows per warp step
    constexpr int NQK = TPL * G;
    constexpr int OUTN = NQK >= W ? NQK / W : 1;
    __shared__ float z_s[G][kChunkTok];
    __shared__ int blk_s[kChunkTok / 16], ntok_s[kChunkTok / 16];
    __shared__ float m_s[G], l_s[G];
    extern __shared__ float o_s[];  // softmax: [kNW][G][D]

    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const ekv_cache &c = a.c;
    const int H = c.num_kv_heads, P = c.page_size, BH = c.batch * H;
    const int CPP = a.CP * P;
    const int cidx = lane % W;
    const long items = (long)BH * a.NC;
    const char *kc = static_cast<const char *>(c.k_cache);
    const char *vc = static_cast<const char *>(c.v_cache);

    for (long it = blockIdx.x; it < items; it += gridDim.x) {
        const int ci = (int)(it / BH), bh = (int)(it % BH);
        const int b = bh / H, h = bh % H;
        int len;
        const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
        int nsel = a.sel_count[bh];
        nsel = nsel < 0 ? 0 : (nsel > a.max_sel ? a.max_sel : nsel);
        if (ci >= (nsel + a.CP - 1) / a.CP) continue;  // uniform over the CTA

        if (tid < a.CP) {
            const int i = ci * a.CP + tid;
            int blk = 0, nt = 0;
            if (i < nsel) {
                const int j = a.sel_idx[(size_t)bh * a.max_sel + i];
                if (j < 0 || j >= np) {
                    flag(c.dev_status, EKV_DEV_BAD_SEL);
                } else {
                    blk = c.page_table[(size_t)b * c.max_pages + j];
                    if (blk < 0 || blk >= c.num_blocks) {
                        flag(c.dev_status, EKV_DEV_BAD_BLOCK);
                        blk = 0;
                    } else {
                        nt = len - j * P < P ? len - j * P : P;
                    }
                }
            }
            blk_s[tid] = blk;
            ntok_s[tid] = nt;
        }
        float qv[G][EPC];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < EPC; ++e)
                qv[g][e] = a.qscale * load_elem<DT>(a.q, ((size_t)b * a.H_q + h * G + g) * D + cidx * EPC + e);
        __syncthreads();

        // ---- logits of the chunk's tokens
        for (int base = warp * TW; base < CPP; base += kNW * TW) {
            uint4 x[TPL];
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
                const int slot = base + i * RPI + lane / W;
                const int pi = slot >> a.Pshift, t = slot & (P - 1);
                x[i] = t < ntok_s[pi]
                           ? ld_stream16(kc + ((((size_t)blk_s[pi] * H + h) * P + t) * D) * ESZ + cidx * 16)
                           : make_uint4(0, 0, 0, 0);
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
                    z_s[g][slot] = t < ntok_s[pi] ? part[r] : -INFINITY;
                }
            }
        }
        __syncthreads();
        if (warp < G) {
            float m = -INFINITY;
            for (int s = lane; s < CPP; s += 32) m = fmaxf(m, z_s[warp][s]);
            m = warp_max(m);
            if (lane == 0) m_s[warp] = m;
        }
        __syncthreads();
        const size_t bq0 = (size_t)b * a.H_q + h * G;

        if constexpr (!SOFTMAX) {
            for (int i = tid; i < G * CPP; i += 256) {
                const int g = i / CPP, s = i - g * CPP;
                a.logits[(bq0 + g) * (size_t)a.LS + (size_t)ci * CPP + s] = z_s[g][s];
            }
            if (tid < G) a.part_ml[((bq0 + tid) * a.NC + ci) * 2] = m_s[tid];
            __syncthreads();
            continue;
        }

        // ---- softmax partial: p = 2^(z - m), l = sum p, o = sum p v
        for (int i = tid; i < G * CPP; i += 256) {
            const int g = i / CPP, s = i - g * CPP;
            const float z = z_s[g][s];
            z_s[g][s] = z == -INFINITY ? 0.f : exp2f(z - m_s[g]);
        }
        __syncthreads();
        if (warp < G) {
            float l = 0.f;
            for (int s = lane; s < CPP; s += 32) l += z_s[warp][s];
            l = warp_sum(l);
            if (lane == 0) l_s[warp] = l;
        }
        float acc[G][EPC];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc[g][e] = 0.f;
        for (int base = warp * TW; base < CPP; base += kNW * TW) {
            uint4 x[TPL];
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
                const int slot = base + i * RPI + lane / W;
                const int pi = slot >> a.Pshift, t = slot & (P - 1);
                x[i] = t < ntok_s[pi]
                           ? ld_stream16(vc + ((((size_t)blk_s[pi] * H + h) * P + t) * D) * ESZ + cidx * 16)
                           : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
                const int slot = base + i * RPI + lane / W;
                float f[EPC];
                Chunk<DT>::unpack(x[i], f);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float p = z_s[g][slot];
#pragma unroll
                    for (int e = 0; e < EPC; ++e) acc[g][e] = fmaf(p, f[e], acc[g][e]);
                }
            }
        }
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
        __syncthreads();
        for (int i = tid; i < G * D; i += 256) {
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
        __syncthreads();
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

template <int DT, int D>
__device__ void finish_entmax(const DecodeArgs &a, int b, int hq, int h, int nsel, int nchunks)
{
    constexpr int CAPW = 256;  // gathered logits per warp
    constexpr int EPC = Chunk<DT>::N;
    constexpr int ESZ = Chunk<DT>::kBytes;
    constexpr int W = D * ESZ / 16;
    constexpr int RPI = 32 / W;
    __shared__ float cz[kNW][CAPW];
    __shared__ int cs[kNW][CAPW];
    __shared__ int cn[kNW];
    __shared__ float red[kNW];
    __shared__ double s_tau;
    __shared__ float o_w[kNW][D];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const ekv_cache &c = a.c;
    const int P = c.page_size;
    const size_t bq = (size_t)b * a.H_q + hq;
    const float *z = a.logits + bq * (size_t)a.LS;
    const bool sparsemax = a.alpha == 2.0f;

    float zmax = -INFINITY;
    for (int ch = tid; ch < nchunks; ch += 256) zmax = fmaxf(zmax, __ldcg(a.part_ml + (bq * a.NC + ch) * 2));
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
    const float thr = zmax - 1.0f;

    // gather the logits above thr: warp w scans a contiguous slot range, in slot order
    const int nslots = nsel * P;
    const int per_warp = ((nslots + kNW - 1) / kNW + 31) / 32 * 32;
    const int s0 = warp * per_warp, s1 = min(s0 + per_warp, nslots);
    int cnt = 0;
    for (int s = s0; s < s1; s += 32) {
        const int sl = s + lane;
        const float v = sl < s1 ? __ldcg(z + sl) : -INFINITY;
        const bool keep = v > thr;
        const unsigned bal = __ballot_sync(kFull, keep);
        const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
        if (keep && pos < CAPW) { cz[warp][pos] = v; cs[warp][pos] = sl; }
        cnt += __popc(bal);
    }
    if (lane == 0) cn[warp] = cnt;
    __syncthreads();
    bool overflow = false;
#pragma unroll
    for (int w = 0; w < kNW; ++w) overflow |= cn[w] > CAPW;

    // threshold: warp 0, Newton from the left, then closed form on the support
    if (warp == 0) {
        auto visit = [&](auto &&fn) {
            if (!overflow) {
                for (int w = 0; w < kNW; ++w)
                    for (int i = lane; i < cn[w]; i += 32) fn(cz[w][i]);
            } else {
                for (int s = lane; s < nslots; s += 32) {
                    const float v = __ldcg(z + s);
                    if (v > thr) fn(v);
                }
            }
        };
        double tau = thr;
#pragma unroll 1
        for (int it = 0; it < 100; ++it) {
            double f = 0.0, df = 0.0;
            visit([&](float v) {
                const double r = (double)v - tau;
                if (r > 0.0) {
                    f += sparsemax ? r : r * r;
                    df += sparsemax ? 1.0 : 2.0 * r;
                }
            });
            f = warp_sum(f) - 1.0;
            df = warp_sum(df);
            if (!(df > 0.0) || !(f > 0.0)) break;
            const double step = f / df;
            if (!(step > 1e-12 * fmax(1.0, fabs(tau)))) break;
            tau += step;
        }
        // exact closed form over the support, until the support is stable
#pragma unroll 1
        for (int round = 0; round < 8; ++round) {
            double n = 0.0, s1v = 0.0;
            visit([&](float v) { if ((double)v > tau) { n += 1.0; s1v += v; } });
            n = warp_sum(n);
            s1v = warp_sum(s1v);
            if (n < 1.0) break;
            double t2;
            if (sparsemax) {
                t2 = (s1v - 1.0) / n;
            } else {
                const double mean = s1v / n;
                double m2 = 0.0;
                visit([&](float v) { if ((double)v > tau) m2 += ((double)v - mean) * ((double)v - mean); });
                m2 = warp_sum(m2);
                const double disc = (1.0 - m2) / n;
                if (disc < 0.0) break;
                t2 = mean - sqrt(disc);
            }
            // stable iff {v > t2} == {v > tau}
            int changed = 0;
            visit([&](float v) { changed |= ((double)v > t2) != ((double)v > tau); });
            changed = __any_sync(kFull, changed);
            tau = t2;
            if (!changed) break;
        }
        if (lane == 0) s_tau = tau;
    }
    __syncthreads();
    const double tau = s_tau;

    // o = sum over the support of p_i v_i; warp w takes its own gathered entries (or, on
    // overflow, every slot s with s % kNW == w)
    const char *vc = static_cast<const char *>(c.v_cache);
    const int H = c.num_kv_heads;
    const int cidx = lane % W, row = lane / W;
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
    const int nmine = overflow ? (nslots + kNW - 1 - warp) / kNW : cn[warp];
    for (int k0 = 0; k0 < nmine; k0 += RPI) {
        const int k = k0 + row;
        float v = -INFINITY;
        int slot = 0;
        if (k < nmine) {
            if (overflow) { slot = warp + k * kNW; v = __ldcg(z + slot); }
            else { slot = cs[warp][k]; v = cz[warp][k]; }
        }
        const double r = (double)v - tau;
        if (r > 0.0) {
            const float p = (float)(sparsemax ? r : r * r);
            const int pi = slot >> a.Pshift, t = slot & (P - 1);
            const int j = a.sel_idx[((size_t)b * H + h) * a.max_sel + pi];
            const int blk = c.page_table[(size_t)b * c.max_pages + j];
            float f[EPC];
            Chunk<DT>::unpack(ld_stream16(vc + ((((size_t)blk * H + h) * P + t) * D) * ESZ + cidx * 16), f);
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc[e] = fmaf(p, f[e], acc[e]);
        }
    }
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
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kNW; ++w) s += o_w[w][i];
        a.out[bq * D + i] = s;
    }
    if (tid == 0) a.stat[bq] = (float)tau;
}

template <int DT, int D, int G, bool SOFTMAX>
__global__ void __launch_bounds__(256)
decode_finish_kernel(DecodeArgs a)
{
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
        pdl_trigger();
        return;
    }
    if constexpr (SOFTMAX) finish_softmax<D>(a, b, hq, nchunks);
    else finish_entmax<DT, D>(a, b, hq, h, nsel, nchunks);
    pdl_trigger();
}

// ------------------------------------------------------------------------------ host side
// Pages per chunk: enough chunks to give every SM a few CTAs, at most 256 tokens per chunk.
int decode_pages_per_chunk(int batch, int H_kv, int max_sel, int P)
{
    long units = (long)batch * H_kv * max_sel;
    long cp = units / (148L * 4);
    const int cap = kChunkTok / P;
    if (cp > cap) cp = cap;
    if (cp < 1) cp = 1;
    return (int)cp;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t decode_workspace_layout(int batch, int H_q, int H_kv, int D, int P, int max_sel,
                               size_t *off_o, size_t *off_logits, int *CP, int *NC)
{
    const int cp = decode_pages_per_chunk(batch, H_kv, max_sel, P);
    const int nc = (max_sel + cp - 1) / cp;
    const size_t BQ = (size_t)batch * H_q;
    size_t off = align256(BQ * nc * 2 * sizeof(float));
    if (off_o) *off_o = off;
    off += align256(BQ * nc * D * sizeof(float));
    if (off_logits) *off_logits = off;
    off += align256(BQ * (size_t)nc * cp * P * sizeof(float));
    if (CP) *CP = cp;
    if (NC) *NC = nc;
    return off;
}

template <int DT, int D, int G>
static cudaError_t launch_decode_t(const DecodeArgs &a, bool softmax, cudaStream_t st, bool pdl)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const long items = (long)a.c.batch * a.c.num_kv_heads * a.NC;
    cudaError_t e;
    if (softmax) {
        auto k = decode_chunk_kernel<DT, D, G, true>;
        cfg.dynamicSmemBytes = sizeof(float) * kNW * G * D;
        const long grid = persistent_grid_size((const void *)k, 256, cfg.dynamicSmemBytes);
        cfg.gridDim = dim3((unsigned)(items < grid ? items : grid));
        e = cudaLaunchKernelEx(&cfg, k, a);
    } else {
        auto k = decode_chunk_kernel<DT, D, G, false>;
        cfg.dynamicSmemBytes = 0;
        const long grid = persistent_grid_size((const void *)k, 256, 0);
        cfg.gridDim = dim3((unsigned)(items < grid ? items : grid));
        e = cudaLaunchKernelEx(&cfg, k, a);
    }
    if (e != cudaSuccess) return e;
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
    size_t off_o, off_logits;
    decode_workspace_layout(c.batch, H_q, c.num_kv_heads, c.head_dim, c.page_size, max_sel,
                            &off_o, &off_logits, &a.CP, &a.NC);
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
