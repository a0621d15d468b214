// tokens.cu -- token-level selection inside the selected pages and attention indexed into the
// paged cache (after the JSSA abstract on ai.info: token-granular selection, one selection per
// KV head, an indexed attention kernel on the standard GQA cache layout with no gather copy).
//
// Step 1 (token_score_kernel): the group score of every candidate token -- the valid tokens of
// the selected pages -- for its KV head, sum_g scale q_g . k = scale (sum_g q_g) . k, in the
// full key space (JSSA fits a low-dimensional scoring subspace to data; with no data the
// subspace is the whole space). Candidate slot i * P + t holds page i of the selection,
// position t; slots past a page's valid tokens hold -inf.
// Step 2 (select_tokens_kernel, select.cu): the T best slots, ties to the lower slot.
// Step 3 (token_attend_kernel): per query head, softmax or exact alpha-entmax over the kept
// tokens, whose K and V rows are read in place through the page table.
#include "decode.cuh"

namespace ekv {

constexpr int kTokRowsSmem = 16384;  // kept tokens whose cache rows the attention keeps on chip
constexpr int kTokPages = 64;        // selected pages per CTA of the token scores, at most

// One CTA per (up to kTokPages selected pages, sequence x KV head). A half-warp scores four
// token rows at a time: lane l of the half reads the 16-byte pieces l (+16) of each row and
// holds the matching coordinates of the group query sum Q = sum_g q_g; the partial dots are
// summed over the half.
template <int DT, int D, int G>
__global__ void __launch_bounds__(256)
token_score_kernel(ekv_cache c, const void *__restrict__ q, int H_q, float scale,
                   const int32_t *__restrict__ sel_idx, const int32_t *__restrict__ sel_count,
                   int max_sel, int ppc, float *__restrict__ tscores)
{
    const int PPC = ppc;  // selected pages per CTA (<= kTokPages)
    constexpr int EPC = Chunk<DT>::N, RB = D * Chunk<DT>::kBytes, W = RB / 16, PPL = (W + 15) / 16;
    constexpr int RIF = 4;  // rows in flight per half-warp
    __shared__ int s_blk[kTokPages], s_nt[kTokPages];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, half = lane >> 4, hl = lane & 15;
    const unsigned hmask = 0xffffu << (16 * half);  // this half-warp's lanes
    const int bh = blockIdx.y, b = bh / c.num_kv_heads, h = bh % c.num_kv_heads;
    const int H = c.num_kv_heads, P = c.page_size;
    pdl_wait();
    int ns = sel_count[bh];
    ns = ns < 0 ? 0 : (ns > max_sel ? max_sel : ns);
    const int i0 = blockIdx.x * PPC;
    if (i0 >= ns) return;
    int len;
    const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
    if (tid < PPC) {
        const int i = i0 + tid;
        int blk = -1, nt = 0;
        if (i < ns) {
            const int j = sel_idx[(size_t)bh * max_sel + i];
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
        }
        s_blk[tid] = blk;
        s_nt[tid] = nt;
    }
    auto owns = [&](int k) { return hl + 16 * k < W; };
    float qv[PPL][EPC];
#pragma unroll
    for (int k = 0; k < PPL; ++k)
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
            float sum = 0.f;
            if (owns(k))
#pragma unroll
                for (int g = 0; g < G; ++g)
                    sum += load_elem<DT>(q, ((size_t)b * H_q + (size_t)h * G + g) * D + (hl + 16 * k) * EPC + e);
            qv[k][e] = sum;
        }
    __syncthreads();
    const int i1 = i0 + PPC < ns ? i0 + PPC : ns;
    const int nrows = (i1 - i0) * P;
    float *out = tscores + (size_t)bh * max_sel * P + (size_t)i0 * P;
    const char *kc = static_cast<const char *>(c.k_cache);
    // the next RIF rows' 16-byte pieces are loaded before the current ones are reduced (kept
    // raw and unpacked row by row), so each half-warp has two groups of rows in flight
    auto fetch = [&](int base, uint4 (&raw)[RIF][PPL], bool (&ok)[RIF]) {
#pragma unroll
        for (int r = 0; r < RIF; ++r) {
            const int rr = base + r, slot = rr / P, t = rr - slot * P;
            ok[r] = rr < nrows && t < s_nt[slot < PPC ? slot : 0];
            const size_t row = ((size_t)(ok[r] ? s_blk[slot] : 0) * H + h) * P + t;
#pragma unroll
            for (int k = 0; k < PPL; ++k)
                raw[r][k] = ok[r] && owns(k) ? ld_stream16(kc + row * RB + (hl + 16 * k) * 16)
                                             : make_uint4(0, 0, 0, 0);
        }
    };
    uint4 cur[RIF][PPL], nxt[RIF][PPL];
    bool okc[RIF], okn[RIF];
    int base = (warp * 2 + half) * RIF;
    if (base < nrows) fetch(base, cur, okc);
    for (; base < nrows; base += 16 * RIF) {
        if (base + 16 * RIF < nrows) fetch(base + 16 * RIF, nxt, okn);
#pragma unroll
        for (int r = 0; r < RIF; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < PPL; ++k) {
                float kf[EPC];
                Chunk<DT>::unpack(cur[r][k], kf);  // zero pieces unpack to 0
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc = fmaf(qv[k][e], kf[e], acc);
            }
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) acc += __shfl_xor_sync(hmask, acc, o);
            if (hl == 0 && base + r < nrows) out[base + r] = okc[r] ? scale * acc : -INFINITY;
        }
#pragma unroll
        for (int r = 0; r < RIF; ++r) {
            okc[r] = okn[r];
#pragma unroll
            for (int k = 0; k < PPL; ++k) cur[r][k] = nxt[r][k];
        }
    }
    pdl_trigger();
}

// One CTA per (sequence, query head), the kept tokens' logits in shared memory.
//   softmax: p = exp(s - max) / sum, stat = log sum exp(s);
//   entmax:  z = (alpha - 1) s; tau by Newton on f(tau)^(alpha-1) = 1, f = sum [z - tau]_+^(1/(alpha-1)),
//            from max z - 1 in fp64, then recomputed in closed form over the support
//            {z > tau} (sparsemax: (sum_S z - 1) / |S|; 1.5-entmax: mean_S - sqrt((1 -
//            sum_S (z - mean_S)^2) / |S|)); p = [z - tau]_+^(1/(alpha-1)), stat = tau.
//   out = sum_i p_i v_i, reading only rows with p_i > 0.
template <int DT, int D, int G>
__global__ void __launch_bounds__(256)
token_attend_kernel(ekv_cache c, const void *__restrict__ q, int H_q, float scale, int attn,
                    const int32_t *__restrict__ tok_page, const int32_t *__restrict__ tok_pos,
                    const int32_t *__restrict__ tok_count, int T, float *__restrict__ out,
                    float *__restrict__ stat)
{
    extern __shared__ float zs[];   // [T] logits, then weights
    __shared__ float qs[D];
    __shared__ double dred[8], dred2[8];
    __shared__ float fred[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hq = blockIdx.x, b = blockIdx.y, h = hq / G;
    const int bh = b * c.num_kv_heads + h;
    const size_t bq = (size_t)b * H_q + hq;
    const int P = c.page_size;
    pdl_wait();
    int n = tok_count[bh];
    n = n < 0 ? 0 : (n > T ? T : n);
    if (n == 0) {
        for (int a = tid; a < D; a += 256) out[bq * D + a] = 0.f;
        if (tid == 0) stat[bq] = -INFINITY;
        return;
    }
    int len;
    const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
    for (int e = tid; e < D; e += 256) qs[e] = load_elem<DT>(q, bq * D + e);
    __syncthreads();
    const int32_t *pg = tok_page + (size_t)bh * T, *ps = tok_pos + (size_t)bh * T;
    auto row_of = [&](int i) -> long long {
        const int j = pg[i], t = ps[i];
        if (j < 0 || j >= np || t < 0 || t >= P || j * P + t >= len) return -1;
        const int blk = c.page_table[(size_t)b * c.max_pages + j];
        if (blk < 0 || blk >= c.num_blocks) return -1;
        return ((long long)blk * c.num_kv_heads + h) * P + t;
    };
    const float alpha = attn == EKV_SOFTMAX ? 1.f : (attn == EKV_ENTMAX15 ? 1.5f : 2.f);
    const float zscale = scale * (attn == EKV_SOFTMAX ? 1.f : alpha - 1.f);
    // the cache row of every kept token, resolved once (all lookups in flight together); for
    // T beyond the shared-memory rows the lookups are repeated where needed
    constexpr int EPC = Chunk<DT>::N, RB = D * Chunk<DT>::kBytes, W = RB / 16, PPL = (W + 15) / 16;
    constexpr int RIF = 4;  // rows in flight per half-warp
    const bool rows_smem = T <= kTokRowsSmem;
    long long *rows = reinterpret_cast<long long *>(zs + ((T + 1) & ~1));  // [T] when rows_smem
    if (rows_smem) {
        for (int i = tid; i < n; i += 256) {
            const long long r = row_of(i);
            if (r < 0) flag(c.dev_status, EKV_DEV_BAD_SEL);
            rows[i] = r;
        }
    } else {
        for (int i = tid; i < n; i += 256)
            if (row_of(i) < 0) flag(c.dev_status, EKV_DEV_BAD_SEL);
    }
    __syncthreads();
    auto row_at = [&](int i) { return rows_smem ? rows[i] : row_of(i); };
    const int half = lane >> 4, hl = lane & 15;
    // the two halves of a warp may take different trip counts through the row loops: their
    // reductions synchronise only their own 16 lanes
    const unsigned hmask = 0xffffu << (16 * half);
    auto owns = [&](int k) { return hl + 16 * k < W; };
    float qv[PPL][EPC];
#pragma unroll
    for (int k = 0; k < PPL; ++k)
#pragma unroll
        for (int e = 0; e < EPC; ++e) qv[k][e] = owns(k) ? qs[(hl + 16 * k) * EPC + e] : 0.f;
    const char *kc = static_cast<const char *>(c.k_cache), *vc = static_cast<const char *>(c.v_cache);
    // logits: a half-warp takes RIF rows at a time, lane l reading pieces l (+16) of each; the
    // next RIF rows' pieces are loaded (kept raw) before the current ones are reduced
    auto fetch = [&](int base, uint4 (&raw)[RIF][PPL], bool (&ok)[RIF]) {
#pragma unroll
        for (int r = 0; r < RIF; ++r) {
            const long long rw = base + r < n ? row_at(base + r) : -1;
            ok[r] = rw >= 0;
#pragma unroll
            for (int k = 0; k < PPL; ++k)
                raw[r][k] = ok[r] && owns(k) ? ld_stream16(kc + (size_t)rw * RB + (hl + 16 * k) * 16)
                                             : make_uint4(0, 0, 0, 0);
        }
    };
    {
        uint4 cur[RIF][PPL], nxt[RIF][PPL];
        bool okc[RIF], okn[RIF];
        int base = (warp * 2 + half) * RIF;
        if (base < n) fetch(base, cur, okc);
        for (; base < n; base += 16 * RIF) {
            if (base + 16 * RIF < n) fetch(base + 16 * RIF, nxt, okn);
#pragma unroll
            for (int r = 0; r < RIF; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < PPL; ++k) {
                    float kf[EPC];
                    Chunk<DT>::unpack(cur[r][k], kf);  // zero pieces unpack to 0
#pragma unroll
                    for (int e = 0; e < EPC; ++e) acc = fmaf(qv[k][e], kf[e], acc);
                }
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) acc += __shfl_xor_sync(hmask, acc, o);
                if (hl == 0 && base + r < n) zs[base + r] = okc[r] ? zscale * acc : -INFINITY;
            }
#pragma unroll
            for (int r = 0; r < RIF; ++r) {
                okc[r] = okn[r];
#pragma unroll
                for (int k = 0; k < PPL; ++k) cur[r][k] = nxt[r][k];
            }
        }
    }
    __syncthreads();
    auto block_max = [&](float v) {
        v = warp_max(v);
        if (lane == 0) fred[warp] = v;
        __syncthreads();
        float m = fred[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) m = fmaxf(m, fred[w]);
        __syncthreads();
        return m;
    };
    auto block_dsum = [&](double v) {
        v = warp_sum(v);
        if (lane == 0) dred[warp] = v;
        __syncthreads();
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += dred[w];
        __syncthreads();
        return s;
    };
    auto block_dsum2 = [&](double &v, double &w) {  // two sums in one round of barriers
        v = warp_sum(v);
        w = warp_sum(w);
        if (lane == 0) { dred[warp] = v; dred2[warp] = w; }
        __syncthreads();
        double s = 0.0, t = 0.0;
#pragma unroll
        for (int k = 0; k < 8; ++k) { s += dred[k]; t += dred2[k]; }
        __syncthreads();
        v = s;
        w = t;
    };
    float mx = -INFINITY;
    for (int i = tid; i < n; i += 256) mx = fmaxf(mx, zs[i]);
    mx = block_max(mx);
    if (mx == -INFINITY) {  // every listed token was out of range (flagged above)
        for (int a = tid; a < D; a += 256) out[bq * D + a] = 0.f;
        if (tid == 0) stat[bq] = -INFINITY;
        return;
    }
    float st;
    if (attn == EKV_SOFTMAX) {
        double l = 0.0;
        for (int i = tid; i < n; i += 256) {
            const float p = zs[i] == -INFINITY ? 0.f : expf(zs[i] - mx);
            zs[i] = p;
            l += p;
        }
        l = block_dsum(l);
        const float inv = (float)(1.0 / l);
        for (int i = tid; i < n; i += 256) zs[i] *= inv;
        st = mx + (float)log(l);
    } else {
        const bool sparse = attn == EKV_SPARSEMAX;
        // Newton on F^(1/p) = 1, F(t) = sum [z - t]_+^p (p = 1 sparsemax, 2 1.5-entmax): F^(1/p)
        // is an l^p norm of (z - t)_+, so it is convex and decreasing, and Newton from
        // t = max z - 1 (where F >= 1) rises monotonically onto the root (for sparsemax F is
        // piecewise linear and the iteration ends once the support is found)
        double lo = (double)mx - 1.0;
        for (int it = 0; it < 64; ++it) {
            double f = 0.0, df = 0.0;
            for (int i = tid; i < n; i += 256) {
                const double r = (double)zs[i] - lo;
                if (r > 0.0) {
                    f += sparse ? r : r * r;
                    df -= sparse ? 1.0 : 2.0 * r;
                }
            }
            block_dsum2(f, df);
            if (!(df < 0.0)) break;
            double step;
            if (sparse) {
                step = (f - 1.0) / -df;
            } else {
                const double rf = sqrt(f);
                step = (rf - 1.0) * 2.0 * rf / -df;
            }
            if (!(step > 1e-13 * fmax(1.0, fabs(lo)))) break;
            lo += step;
        }
        // closed form over the support {z > lo}
        double s1 = 0.0, s2 = 0.0, k = 0.0;
        for (int i = tid; i < n; i += 256) {
            if ((double)zs[i] > lo) { s1 += zs[i]; s2 += (double)zs[i] * zs[i]; k += 1.0; }
        }
        s1 = block_dsum(s1);
        s2 = block_dsum(s2);
        k = block_dsum(k);
        double tau;
        if (sparse) {
            tau = (s1 - 1.0) / k;
        } else {
            const double mean = s1 / k, ss = s2 - k * mean * mean;
            const double disc = (1.0 - ss) / k;
            tau = mean - sqrt(disc > 0.0 ? disc : 0.0);
        }
        for (int i = tid; i < n; i += 256) {
            const double r = (double)zs[i] - tau;
            zs[i] = r > 0.0 ? (float)(sparse ? r : r * r) : 0.f;
        }
        st = (float)tau;
    }
    __syncthreads();
    // out = sum p_i v_i over the rows with p_i > 0: a half-warp takes RIF rows at a time, each
    // lane accumulating its coordinates; then the halves and the warps are summed in order
    float acc[PPL][EPC];
#pragma unroll
    for (int k = 0; k < PPL; ++k)
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[k][e] = 0.f;
    for (int base = (warp * 2 + half) * RIF; base < n; base += 16 * RIF) {
        float vf[RIF][PPL][EPC], pr[RIF];
#pragma unroll
        for (int r = 0; r < RIF; ++r) {
            pr[r] = base + r < n ? zs[base + r] : 0.f;
            const long long rw = pr[r] != 0.f ? row_at(base + r) : -1;
#pragma unroll
            for (int k = 0; k < PPL; ++k) {
                if (rw >= 0 && owns(k)) {
                    Chunk<DT>::unpack(ld_stream16(vc + (size_t)rw * RB + (hl + 16 * k) * 16), vf[r][k]);
                } else {
#pragma unroll
                    for (int e = 0; e < EPC; ++e) vf[r][k][e] = 0.f;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RIF; ++r)
#pragma unroll
            for (int k = 0; k < PPL; ++k)
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[k][e] = fmaf(pr[r], vf[r][k][e], acc[k][e]);
    }
    __shared__ float opart[8][D];
#pragma unroll
    for (int k = 0; k < PPL; ++k)
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[k][e] += __shfl_xor_sync(kFull, acc[k][e], 16);
    if (half == 0) {
#pragma unroll
        for (int k = 0; k < PPL; ++k)
            if (owns(k))
#pragma unroll
                for (int e = 0; e < EPC; ++e) opart[warp][(hl + 16 * k) * EPC + e] = acc[k][e];
    }
    __syncthreads();
    for (int a = tid; a < D; a += 256) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += opart[w][a];
        out[bq * D + a] = sum;
    }
    if (tid == 0) stat[bq] = st;
}

template <int DT, int D, int G>
static cudaError_t launch_tokens_t(const ekv_cache &c, const void *q, int H_q, float scale,
                                   const int32_t *sel_idx, const int32_t *sel_count, int max_sel,
                                   float *tscores, cudaStream_t st)
{
    // pages per CTA: the most (up to kTokPages) that still give 3 CTAs per SM (of the 4 that fit),
    // so that each CTA's page resolution is spent on a longer run of rows
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long pairs = (long long)c.batch * c.num_kv_heads;
    int ppc = kTokPages;
    while (ppc > 8 && (long long)((max_sel + ppc - 1) / ppc) * pairs < 3ll * sms) ppc >>= 1;
    const dim3 grid((max_sel + ppc - 1) / ppc, c.batch * c.num_kv_heads);
    token_score_kernel<DT, D, G><<<grid, 256, 0, st>>>(c, q, H_q, scale, sel_idx, sel_count, max_sel,
                                                        ppc, tscores);
    return cudaGetLastError();
}

template <int DT, int D, int G>
static cudaError_t launch_attend_t(const ekv_cache &c, const void *q, int H_q, float scale, int attn,
                                   const int32_t *tok_page, const int32_t *tok_pos,
                                   const int32_t *tok_count, int T, float *out, float *stat,
                                   cudaStream_t st)
{
    auto k = token_attend_kernel<DT, D, G>;
    // the logits, then (up to kTokRowsSmem tokens) the kept tokens' cache rows
    const size_t smem = sizeof(float) * (size_t)((T + 1) & ~1) +
                        (T <= kTokRowsSmem ? sizeof(long long) * (size_t)T : 0);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k<<<dim3(H_q, c.batch), 256, smem, st>>>(c, q, H_q, scale, attn, tok_page, tok_pos, tok_count, T, out, stat);
    return cudaGetLastError();
}

#define EKV_TOKEN_DISPATCH(FN, ...)                                                               \
    do {                                                                                          \
        const int G = H_q / c.num_kv_heads;                                                       \
        if (c.dtype == EKV_BF16) {                                                                \
            if (c.head_dim == 128) {                                                              \
                switch (G) {                                                                      \
                case 1: return FN<EKV_BF16, 128, 1>(__VA_ARGS__);                                 \
                case 2: return FN<EKV_BF16, 128, 2>(__VA_ARGS__);                                 \
                case 4: return FN<EKV_BF16, 128, 4>(__VA_ARGS__);                                 \
                default: return FN<EKV_BF16, 128, 8>(__VA_ARGS__);                                \
                }                                                                                 \
            }                                                                                     \
            switch (G) {                                                                          \
            case 1: return FN<EKV_BF16, 64, 1>(__VA_ARGS__);                                      \
            case 2: return FN<EKV_BF16, 64, 2>(__VA_ARGS__);                                      \
            case 4: return FN<EKV_BF16, 64, 4>(__VA_ARGS__);                                      \
            default: return FN<EKV_BF16, 64, 8>(__VA_ARGS__);                                     \
            }                                                                                     \
        }                                                                                         \
        if (c.head_dim == 128) {                                                                  \
            switch (G) {                                                                          \
            case 1: return FN<EKV_F32, 128, 1>(__VA_ARGS__);                                      \
            case 2: return FN<EKV_F32, 128, 2>(__VA_ARGS__);                                      \
            case 4: return FN<EKV_F32, 128, 4>(__VA_ARGS__);                                      \
            default: return FN<EKV_F32, 128, 8>(__VA_ARGS__);                                     \
            }                                                                                     \
        }                                                                                         \
        switch (G) {                                                                              \
        case 1: return FN<EKV_F32, 64, 1>(__VA_ARGS__);                                           \
        case 2: return FN<EKV_F32, 64, 2>(__VA_ARGS__);                                           \
        case 4: return FN<EKV_F32, 64, 4>(__VA_ARGS__);                                           \
        default: return FN<EKV_F32, 64, 8>(__VA_ARGS__);                                          \
        }                                                                                         \
    } while (0)

cudaError_t launch_token_scores(const ekv_cache &c, const void *q, int H_q, float scale,
                                const int32_t *sel_idx, const int32_t *sel_count, int max_sel,
                                float *tscores, cudaStream_t st)
{
    EKV_TOKEN_DISPATCH(launch_tokens_t, c, q, H_q, scale, sel_idx, sel_count, max_sel, tscores, st);
}

cudaError_t launch_token_attend(const ekv_cache &c, const void *q, int H_q, float scale, int attn,
                                const int32_t *tok_page, const int32_t *tok_pos,
                                const int32_t *tok_count, int T, float *out, float *stat,
                                cudaStream_t st)
{
    EKV_TOKEN_DISPATCH(launch_attend_t, c, q, H_q, scale, attn, tok_page, tok_pos, tok_count, T,
                       out, stat, st);
}

#undef EKV_TOKEN_DISPATCH

}  // namespace ekv
