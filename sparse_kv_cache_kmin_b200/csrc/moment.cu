// moment.cu -- moment correction of a sparse softmax decode for the pages a step skips
// (MomentKV technical summary, gist.science: Methodology §1 compact moment statistics, §2
// first-order estimate of the evicted output, §4 normalisation-corrected mix).
//
// The cache keeps every token; a decode step skips the pages it did not select, and those
// tokens play the part of MomentKV's evicted set E. Per (sequence, KV head) the library keeps
// running sums over every token appended so far, in one fp32 record of EKV_MOMENT_FLOATS(d)
// floats: { n, 0, 0, 0, sum k [d], sum v [d], sum v k^T [d][d] (row a: value coordinate) }.
// E's sums are the running sums less those of the selected tokens, which the decode re-reads:
//   n_R, sum_R k, sum_R v and, per query g, u_g = sum_R v (k . q_g).
// Then per query (logits s = scale q.k):
//   n_e = n - n_R,  kbar = (sum k - sum_R k) / n_e,  vbar = (sum v - sum_R v) / n_e,
//   sum_E v (k.q) = (sum v k^T) q - u_g,
//   St q = sum_E (v - vbar)(k - kbar)^T q = sum_E v (k.q) - n_e vbar (kbar.q),
//   fE = vbar + (scale / n_e) St q,           (first-order expansion around scale q.kbar)
//   log ZE = log n_e + scale q.kbar,          (Jensen lower bound on E's partition sum)
//   out = wR fR + (1 - wR) fE,  wR = ZR / (ZR + ZE),  stat = log(ZR + ZE),
// where fR and log ZR are the plain softmax output and log-partition over the selected pages.
#include "decode.cuh"

namespace ekv {

constexpr int kMomTok = 4096;  // tokens per CTA of the running-sum update
constexpr int kMomSub = 32;    // tokens staged in shared memory at a time
constexpr int kRetPages = 64;  // selected pages per CTA of the retained sums, at most

__host__ __device__ constexpr int moment_floats(int d) { return EKV_MOMENT_FLOATS(d); }
__host__ __device__ constexpr int retained_floats(int d, int G) { return 4 + 2 * d + G * d; }

// Running sums over the appended tokens [new_start[b], new_start[b] + new_count[b]) of every
// (sequence, KV head): one CTA per (4096-token slice, KV head, sequence). A thread owns a
// (d/16) x (d/16) block of sum v k^T (rows (tid / 16) * d/16.., columns (tid % 16) * d/16..),
// threads 0..d-1 the key sums and d..2d-1 the value sums; the slice's partial sums are added
// to the record with atomics.
template <int DT, int D>
__global__ void __launch_bounds__(256)
moment_update_kernel(ekv_cache c, float *__restrict__ moments, const int32_t *__restrict__ new_start,
                     const int32_t *__restrict__ new_count, int max_new)
{
    constexpr int RB = D / 16;
    __shared__ float ks[kMomSub][D], vs[kMomSub][D];
    __shared__ long long row_s[kMomSub];  // cache row of each staged token, -1: none
    const int tid = threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    const int P = c.page_size, H = c.num_kv_heads;
    int len;
    seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
    int s = new_start[b], n = new_count[b];
    if (n <= 0) return;
    if (s < 0 || s + n > len || n > max_new) {
        if (blockIdx.x == 0 && h == 0 && tid == 0) flag(c.dev_status, EKV_DEV_BAD_RANGE);
        s = s < 0 ? 0 : (s > len ? len : s);
        const int e = s + n > len ? len : s + n;
        n = e - s > max_new ? max_new : e - s;
        if (n <= 0) return;
    }
    const int t0 = s + blockIdx.x * kMomTok;
    const int t1 = t0 + kMomTok < s + n ? t0 + kMomTok : s + n;
    if (t0 >= t1) return;

    const int a0 = (tid / 16) * RB, c0 = (tid % 16) * RB;
    float acc[RB][RB];
#pragma unroll
    for (int i = 0; i < RB; ++i)
#pragma unroll
        for (int j = 0; j < RB; ++j) acc[i][j] = 0.f;
    float lin = 0.f;  // threads 0..D-1: sum k[tid]; D..2D-1: sum v[tid - D]
    int counted = 0;
    for (int u0 = t0; u0 < t1; u0 += kMomSub) {
        if (tid < kMomSub) {
            long long row = -1;
            const int t = u0 + tid;
            if (t < t1) {
                const int blk = c.page_table[(size_t)b * c.max_pages + t / P];
                if (blk < 0 || blk >= c.num_blocks) flag(c.dev_status, EKV_DEV_BAD_BLOCK);
                else row = ((long long)blk * H + h) * P + t % P;
            }
            row_s[tid] = row;
        }
        __syncthreads();
        for (int i = tid; i < kMomSub * D; i += 256) {
            const int tt = i / D, cc = i % D;
            const long long row = row_s[tt];
            ks[tt][cc] = row >= 0 ? load_elem<DT>(c.k_cache, (size_t)row * D + cc) : 0.f;
            vs[tt][cc] = row >= 0 ? load_elem<DT>(c.v_cache, (size_t)row * D + cc) : 0.f;
        }
        __syncthreads();
        for (int tt = 0; tt < kMomSub; ++tt) {
            if (row_s[tt] < 0) continue;
            ++counted;
            float vv[RB], kk[RB];
#pragma unroll
            for (int i = 0; i < RB; ++i) { vv[i] = vs[tt][a0 + i]; kk[i] = ks[tt][c0 + i]; }
#pragma unroll
            for (int i = 0; i < RB; ++i)
#pragma unroll
                for (int j = 0; j < RB; ++j) acc[i][j] = fmaf(vv[i], kk[j], acc[i][j]);
            if (tid < D) lin += ks[tt][tid];
            else if (tid < 2 * D) lin += vs[tt][tid - D];
        }
        __syncthreads();
    }
    float *rec = moments + ((size_t)b * H + h) * moment_floats(D);
    if (tid == 0) atomicAdd(rec, (float)counted);
    if (tid < 2 * D) atomicAdd(rec + 4 + tid, lin);
    float *S = rec + 4 + 2 * D;
#pragma unroll
    for (int i = 0; i < RB; ++i)
#pragma unroll
        for (int j = 0; j < RB; ++j) atomicAdd(S + (size_t)(a0 + i) * D + c0 + j, acc[i][j]);
}

// Sums over the selected tokens of one (sequence, KV head), up to kRetPages selected pages per CTA:
// n_R, sum_R k, sum_R v and u_g = sum_R v (k . q_g) for the G queries, added with atomics to a
// zeroed [B * H_kv][retained_floats(d, G)] region. A half-warp takes one token row at a time:
// lane l of the half reads the 16-byte pieces l of the K and V rows (8 coordinates each), the
// G dot products k . q_g are summed over the half's lanes, and each lane keeps its coordinates
// of sum k, sum v and u_g in registers; the CTA adds its partial sums once at the end.
template <int DT, int D, int G>
__global__ void __launch_bounds__(256, G <= 4 ? 2 : 1)  // G <= 4: two CTAs per SM
moment_retained_kernel(ekv_cache c, const void *__restrict__ q, int H_q,
                       const int32_t *__restrict__ sel_idx, const int32_t *__restrict__ sel_count,
                       int max_sel, int ppc, float *__restrict__ ret)
{
    const int PPC = ppc;                           // selected pages per CTA (<= kRetPages)
    constexpr int EPC = Chunk<DT>::N;              // coordinates per 16-byte piece
    constexpr int W = D * Chunk<DT>::kBytes / 16;  // pieces per row
    constexpr int PPL = (W + 15) / 16;             // pieces per lane of a half-warp
    __shared__ int s_blk[kRetPages], s_nt[kRetPages];
    __shared__ float red[8][2 * D + G * D];
    __shared__ int s_cnt[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int half = lane >> 4, hl = lane & 15;
    const unsigned hmask = 0xffffu << (16 * half);  // this half-warp's lanes
    const int bh = blockIdx.y, b = bh / c.num_kv_heads, h = bh % c.num_kv_heads;
    const int P = c.page_size;
    int ns = sel_count[bh];
    ns = ns < 0 ? 0 : (ns > max_sel ? max_sel : ns);
    const int i0 = blockIdx.x * PPC;
    if (i0 >= ns) return;
    int len;
    const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
    if (tid < PPC) {  // an invalid page or selection counts nothing; the decode flags it
        const int i = i0 + tid;
        int blk = -1, nt = 0;
        if (i < ns) {
            const int j = sel_idx[(size_t)bh * max_sel + i];
            if (j >= 0 && j < np) {
                blk = c.page_table[(size_t)b * c.max_pages + j];
                if (blk >= 0 && blk < c.num_blocks) nt = len - j * P < P ? len - j * P : P;
                else blk = -1;
            }
        }
        s_blk[tid] = blk;
        s_nt[tid] = nt;
    }
    // lane hl of a half-warp owns pieces hl + 16 k (k < PPL) of a row: coordinates
    // [(hl + 16 k) * EPC, (hl + 16 k + 1) * EPC)
    auto owns = [&](int k) { return hl + 16 * k < W; };
    float qv[G][PPL][EPC];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int k = 0; k < PPL; ++k)
#pragma unroll
            for (int e = 0; e < EPC; ++e)
                qv[g][k][e] = owns(k) ? load_elem<DT>(q, ((size_t)b * H_q + (size_t)h * G + g) * D +
                                                             (hl + 16 * k) * EPC + e)
                                      : 0.f;
    float sk[PPL][EPC], sv[PPL][EPC], u[G][PPL][EPC];
#pragma unroll
    for (int k = 0; k < PPL; ++k)
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
            sk[k][e] = 0.f;
            sv[k][e] = 0.f;
#pragma unroll
            for (int g = 0; g < G; ++g) u[g][k][e] = 0.f;
        }
    int counted = 0;
    __syncthreads();
    const char *kc = static_cast<const char *>(c.k_cache), *vc = static_cast<const char *>(c.v_cache);
    constexpr int RB = D * Chunk<DT>::kBytes;
    // the next row's 16-byte pieces are loaded before this row is reduced, so each half-warp
    // keeps a row in flight while it computes (every half takes the same PPC * P / 16 rows)
    auto fetch = [&](int rho, uint4 (&kr)[PPL], uint4 (&vr)[PPL]) {
        const int slot = rho / P, t = rho - slot * P;
        const bool valid = t < s_nt[slot];
        const size_t row = ((size_t)(valid ? s_blk[slot] : 0) * c.num_kv_heads + h) * P + t;
#pragma unroll
        for (int k = 0; k < PPL; ++k) {
            if (valid && owns(k)) {
                kr[k] = ld_stream16(kc + row * RB + (hl + 16 * k) * 16);
                vr[k] = ld_stream16(vc + row * RB + (hl + 16 * k) * 16);
            } else {
                kr[k] = make_uint4(0, 0, 0, 0);
                vr[k] = make_uint4(0, 0, 0, 0);
            }
        }
        return valid;
    };
    uint4 kr[PPL], vr[PPL];
    bool valid_next = fetch(warp * 2 + half, kr, vr);
    for (int rho = warp * 2 + half; rho < PPC * P; rho += 16) {
        const bool valid = valid_next;
        float kf[PPL][EPC], vf[PPL][EPC];
#pragma unroll
        for (int k = 0; k < PPL; ++k) {
            Chunk<DT>::unpack(kr[k], kf[k]);  // zero pieces unpack to 0
            Chunk<DT>::unpack(vr[k], vf[k]);
        }
        if (rho + 16 < PPC * P) valid_next = fetch(rho + 16, kr, vr);
        float dot[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < PPL; ++k)
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc = fmaf(qv[g][k][e], kf[k][e], acc);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) acc += __shfl_xor_sync(hmask, acc, o);
            dot[g] = acc;
        }
#pragma unroll
        for (int k = 0; k < PPL; ++k)
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                sk[k][e] += kf[k][e];
                sv[k][e] += vf[k][e];
#pragma unroll
                for (int g = 0; g < G; ++g) u[g][k][e] = fmaf(vf[k][e], dot[g], u[g][k][e]);
            }
        counted += valid;
    }
    // the two half-warps' rows, then the warps
#pragma unroll
    for (int k = 0; k < PPL; ++k)
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
            sk[k][e] += __shfl_xor_sync(kFull, sk[k][e], 16);
            sv[k][e] += __shfl_xor_sync(kFull, sv[k][e], 16);
#pragma unroll
            for (int g = 0; g < G; ++g) u[g][k][e] += __shfl_xor_sync(kFull, u[g][k][e], 16);
        }
    counted += __shfl_xor_sync(kFull, counted, 16);
    if (half == 0) {
#pragma unroll
        for (int k = 0; k < PPL; ++k) {
            if (!owns(k)) continue;
            const int c0 = (hl + 16 * k) * EPC;
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                red[warp][c0 + e] = sk[k][e];
                red[warp][D + c0 + e] = sv[k][e];
#pragma unroll
                for (int g = 0; g < G; ++g) red[warp][2 * D + g * D + c0 + e] = u[g][k][e];
            }
        }
    }
    if (lane == 0) s_cnt[warp] = counted;
    __syncthreads();
    float *r = ret + (size_t)bh * retained_floats(D, G);
    for (int i = tid; i < 2 * D + G * D; i += 256) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += red[w][i];
        atomicAdd(r + 4 + i, sum);
    }
    if (tid == 0) {
        int n = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) n += s_cnt[w];
        atomicAdd(r, (float)n);
    }
}

// One CTA per (sequence, query head): turns the plain softmax result over the selected pages
// (out, stat) into the moment-corrected one, in place.
template <int DT, int D, int G>
__global__ void __launch_bounds__(256)
moment_correct_kernel(ekv_cache c, const float *__restrict__ moments, const void *__restrict__ q,
                      int H_q, float scale, const float *__restrict__ ret, float *__restrict__ out,
                      float *__restrict__ stat)
{
    __shared__ float qs[D], kbar[D], vbar[D], sq[D], red[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hq = blockIdx.x, b = blockIdx.y, h = hq / G, g = hq % G;
    const size_t bh = (size_t)b * c.num_kv_heads + h, bq = (size_t)b * H_q + hq;
    const float *rec = moments + bh * moment_floats(D);
    const float *r = ret + bh * retained_floats(D, G);
    // (sum v k^T) q: warp w takes rows a = w, w + 8, ... (D / 8 of them), lane l coordinates
    // l, l + 32, ...; every row's loads are issued first, before anything else of the
    // correction, so they are in flight together and overlap the steps below
    const float *S = rec + 4 + 2 * D;
    constexpr int RPW = D / 8, CPL = D / 32;
    float sv[RPW][CPL];
#pragma unroll
    for (int i = 0; i < RPW; ++i)
#pragma unroll
        for (int k = 0; k < CPL; ++k) sv[i][k] = __ldg(S + (size_t)(warp + 8 * i) * D + lane + 32 * k);
    const float n_e = rec[0] - r[0];
    if (!(n_e >= 0.5f)) return;  // nothing skipped: the plain softmax stands
    for (int i = tid; i < D; i += 256) {
        qs[i] = load_elem<DT>(q, bq * D + i);
        kbar[i] = (rec[4 + i] - r[4 + i]) / n_e;
        vbar[i] = (rec[4 + D + i] - r[4 + D + i]) / n_e;
    }
    __syncthreads();
    // kbar . q
    float part = tid < D ? kbar[tid] * qs[tid] : 0.f;
    part = warp_sum(part);
    if (lane == 0) red[warp] = part;
    __syncthreads();
    float qk = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) qk += red[w];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < CPL; ++k) acc = fmaf(sv[i][k], qs[lane + 32 * k], acc);
        acc = warp_sum(acc);
        const int a = warp + 8 * i;
        if (lane == 0) sq[a] = acc - r[4 + 2 * D + g * D + a];  // sum_E v (k.q)
    }
    __syncthreads();
    const float lzr = stat[bq];  // -inf when nothing is selected
    const float lze = logf(n_e) + scale * qk;
    const float m = lzr > lze ? lzr : lze;
    const float zr = expf(lzr - m), ze = expf(lze - m);
    const float wr = zr / (zr + ze);
    for (int a = tid; a < D; a += 256) {
        const float stq = sq[a] - n_e * vbar[a] * qk;
        const float fe = vbar[a] + scale / n_e * stq;
        out[bq * D + a] = wr * out[bq * D + a] + (1.f - wr) * fe;
    }
    if (tid == 0) stat[bq] = m + logf(zr + ze);
}

size_t moment_retained_bytes(int batch, int H_kv, int D, int G)
{
    return (size_t)batch * H_kv * retained_floats(D, G) * sizeof(float);
}

template <int DT, int D>
static cudaError_t launch_update_t(const ekv_cache &c, float *moments, const int32_t *new_start,
                                   const int32_t *new_count, int max_new, cudaStream_t st)
{
    const dim3 grid((max_new + kMomTok - 1) / kMomTok, c.num_kv_heads, c.batch);
    moment_update_kernel<DT, D><<<grid, 256, 0, st>>>(c, moments, new_start, new_count, max_new);
    return cudaGetLastError();
}

cudaError_t launch_moment_update(const ekv_cache &c, float *moments, const int32_t *new_start,
                                 const int32_t *new_count, int max_new, cudaStream_t st)
{
    if (max_new <= 0) return cudaSuccess;
    if (c.dtype == EKV_BF16)
        return c.head_dim == 128 ? launch_update_t<EKV_BF16, 128>(c, moments, new_start, new_count, max_new, st)
                                 : launch_update_t<EKV_BF16, 64>(c, moments, new_start, new_count, max_new, st);
    return c.head_dim == 128 ? launch_update_t<EKV_F32, 128>(c, moments, new_start, new_count, max_new, st)
                             : launch_update_t<EKV_F32, 64>(c, moments, new_start, new_count, max_new, st);
}

template <int DT, int D, int G>
static cudaError_t launch_correct_t(const ekv_cache &c, const float *moments, const void *q,
                                    int H_q, float scale, const int32_t *sel_idx,
                                    const int32_t *sel_count, int max_sel, float *ret,
                                    float *out, float *stat, cudaStream_t st, bool after_decode)
{
    if (!after_decode) {  // retained sums (before the decode, which does not depend on them)
        cudaError_t e = cudaMemsetAsync(ret, 0, moment_retained_bytes(c.batch, c.num_kv_heads, D, G), st);
        if (e != cudaSuccess) return e;
        // pages per CTA: the most (up to kRetPages) that still give 1.5 CTAs per SM, so that long
        // per-CTA row loops keep the loads flowing without leaving SMs idle
        int dev = 0, sms = 0;
        e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        const long long pairs = (long long)c.batch * c.num_kv_heads;
        int ppc = kRetPages;
        while (ppc > 8 && (long long)((max_sel + ppc - 1) / ppc) * pairs * 2 < 3ll * sms) ppc >>= 1;
        const dim3 grid((max_sel + ppc - 1) / ppc, c.batch * c.num_kv_heads);
        moment_retained_kernel<DT, D, G><<<grid, 256, 0, st>>>(c, q, H_q, sel_idx, sel_count, max_sel,
                                                               ppc, ret);
        return cudaGetLastError();
    }
    moment_correct_kernel<DT, D, G><<<dim3(H_q, c.batch), 256, 0, st>>>(c, moments, q, H_q, scale, ret, out, stat);
    return cudaGetLastError();
}

template <int DT, int D>
static cudaError_t launch_correct_g(const ekv_cache &c, const float *moments, const void *q, int H_q,
                                    float scale, const int32_t *sel_idx, const int32_t *sel_count,
                                    int max_sel, float *ret, float *out, float *stat,
                                    cudaStream_t st, bool after_decode)
{
    switch (H_q / c.num_kv_heads) {
    case 1: return launch_correct_t<DT, D, 1>(c, moments, q, H_q, scale, sel_idx, sel_count, max_sel, ret, out, stat, st, after_decode);
    case 2: return launch_correct_t<DT, D, 2>(c, moments, q, H_q, scale, sel_idx, sel_count, max_sel, ret, out, stat, st, after_decode);
    case 4: return launch_correct_t<DT, D, 4>(c, moments, q, H_q, scale, sel_idx, sel_count, max_sel, ret, out, stat, st, after_decode);
    default: return launch_correct_t<DT, D, 8>(c, moments, q, H_q, scale, sel_idx, sel_count, max_sel, ret, out, stat, st, after_decode);
    }
}

// Before the decode (after_decode = false): zero the retained-sum region and fill it. After
// the decode (true): correct out / stat in place.
cudaError_t launch_moment_pass(const ekv_cache &c, const float *moments, const void *q, int H_q,
                               float scale, const int32_t *sel_idx, const int32_t *sel_count,
                               int max_sel, float *ret, float *out, float *stat, cudaStream_t st,
                               bool after_decode)
{
    if (c.dtype == EKV_BF16)
        return c.head_dim == 128
                   ? launch_correct_g<EKV_BF16, 128>(c, moments, q, H_q, scale, sel_idx, sel_count, max_sel, ret, out, stat, st, after_decode)
                   : launch_correct_g<EKV_BF16, 64>(c, moments, q, H_q, scale, sel_idx, sel_count, max_sel, ret, out, stat, st, after_decode);
    return c.head_dim == 128
               ? launch_correct_g<EKV_F32, 128>(c, moments, q, H_q, scale, sel_idx, sel_count, max_sel, ret, out, stat, st, after_decode)
               : launch_correct_g<EKV_F32, 64>(c, moments, q, H_q, scale, sel_idx, sel_count, max_sel, ret, out, stat, st, after_decode);
}

}  // namespace ekv
