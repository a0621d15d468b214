/*
 * ekv_oracle.c -- plain, slow CPU oracle for query-aware sparse decode over a paged KV cache.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the CPU-baseline leg
 * of the benchmark may load this library; the product path never calls it, and this file
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it follows ("EntmaxKV: support-aware decoding for alpha-entmax attention", technical
 * summary on gist.science):
 *   §2     the KV cache is split into pages; decoding reads whole pages;
 *   §2.A   per-page metadata: coordinate-wise key minimum/maximum (a bounding box) giving a
 *          deterministic upper bound on the best attention score any token of the page can
 *          reach for a query; per-page first and second key moments (mean, variance) so that
 *          a page's token scores can be modelled as a Gaussian;
 *   §2.B.1 fixed-budget selection of the k pages with the largest upper bounds;
 *   §2.B.2 Gaussian-aware selection: solve an approximate entmax normalisation equation for a
 *          threshold tau-hat, keep pages whose estimated maximum score clears tau-hat less a
 *          safety margin Delta;
 *   §2.C   exact alpha-entmax attention over the selected pages only (softmax for the
 *          comparison the summary draws in §1 and §3).
 * And, for softmax over a page selection, the moment correction for the skipped tokens of the
 * MomentKV technical summary (gist.science), Methodology §1, §2, §4 (ora_moment_corrected_head);
 * token-level selection inside the selected pages with indexed attention, after the JSSA
 * abstract (ai.info) (ora_token_topk_head, ora_attend_tokens_head). Their readings are stated
 * at the functions.
 * Readings of points the summary leaves open (all stated again in the design notes):
 *   - logits are s = scale * q.k, with scale an argument;
 *   - alpha-entmax: p_i = [(alpha-1) z_i - tau]_+^(1/(alpha-1)) with sum p = 1, written here
 *     in the z = (alpha-1) s domain as p_i = [z_i - tau]_+^(1/(alpha-1));
 *   - a GQA group of G query heads shares one KV head; the top-k page score is the sum of the
 *     G per-query bounds; the Gaussian policy solves tau-hat per query and keeps the union;
 *   - the "estimated maximum score" of §2.B.2 is the bounding-box bound itself; a second
 *     reading, the Gaussian estimate of a page's maximum capped by that bound,
 *     min(UB, m + sqrt(2 ln n_j) sqrt(v)), is offered beside it (ora_gauss_select_est);
 *   - the margin is in the z domain: keep page j iff (alpha-1)*UB > tau-hat - Delta;
 *   - page variance is per coordinate and population (divide by the count n);
 *   - the approximate normalisation equation replaces each page's n_j token scores by n_j
 *     independent draws from N(m, v) and asks that the expected entmax mass be one;
 *   - only tokens t < seq_len exist; a partly filled last page holds fewer than P tokens;
 *   - top-k ties go to the lower page index; selections are emitted in ascending page order.
 *
 * All arithmetic is float64. bf16 inputs are widened exactly (a bf16 value is the upper half
 * of an IEEE float32).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_F32 0
#define ORA_BF16 1

#define ORA_SOFTMAX 0
#define ORA_ENTMAX15 1
#define ORA_SPARSEMAX 2

/* Exact widening of one stored element to double. */
static double elem(const void *base, int dtype, size_t i)
{
    if (dtype == ORA_F32)
        return (double)((const float *)base)[i];
    uint32_t w = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* Offset of element (block, head, token-in-page, coordinate) in the paged layout
 * [num_blocks][H_kv][P][d]. */
static size_t cache_off(int block, int h, int t, int c, int H_kv, int P, int d)
{
    return (((size_t)block * H_kv + h) * P + t) * d + c;
}

static int pages_of(int seq_len, int P) { return (seq_len + P - 1) / P; }

/* ---------------------------------------------------------------------------------------
 * §2.A page metadata, computed from scratch over each page's valid tokens.
 * Outputs are indexed by logical page j of the sequence: [N_p][d].
 * kmin/kmax: coordinate-wise minimum/maximum of the keys; mean: arithmetic mean;
 * var: population variance, two-pass. Returns the page count, or -1 on a page-table entry
 * outside [0, num_blocks).
 * ------------------------------------------------------------------------------------- */
int ora_page_meta_head(const void *k_cache, int dtype, int num_blocks, int H_kv, int P, int d,
                       const int32_t *pt_row, int seq_len, int h,
                       double *kmin, double *kmax, double *mean, double *var)
{
    int n_pages = pages_of(seq_len, P);
    for (int j = 0; j < n_pages; ++j) {
        int block = pt_row[j];
        if (block < 0 || block >= num_blocks)
            return -1;
        int n = seq_len - j * P < P ? seq_len - j * P : P;
        for (int c = 0; c < d; ++c) {
            double lo = INFINITY, hi = -INFINITY, sum = 0.0;
            for (int t = 0; t < n; ++t) {
                double x = elem(k_cache, dtype, cache_off(block, h, t, c, H_kv, P, d));
                if (x < lo) lo = x;
                if (x > hi) hi = x;
                sum += x;
            }
            double mu = sum / n;
            double ss = 0.0;
            for (int t = 0; t < n; ++t) {
                double x = elem(k_cache, dtype, cache_off(block, h, t, c, H_kv, P, d));
                ss += (x - mu) * (x - mu);
            }
            kmin[(size_t)j * d + c] = lo;
            kmax[(size_t)j * d + c] = hi;
            if (mean) mean[(size_t)j * d + c] = mu;
            if (var) var[(size_t)j * d + c] = ss / n;
        }
    }
    return n_pages;
}

/* ---------------------------------------------------------------------------------------
 * §2.A deterministic page bound, evaluated literally:
 *   UB_{g,j} = scale * sum_c max(q_{g,c} * kmin_{j,c}, q_{g,c} * kmax_{j,c})
 * and the GQA group score used by top-k: S_j = sum_g UB_{g,j}.
 * q: [G][d]; kmin/kmax: [n_pages][d]; ub: [G][n_pages] (may be NULL); S: [n_pages] (may be NULL).
 * ------------------------------------------------------------------------------------- */
void ora_score_head(const double *q, int G, int d, double scale,
                    const double *kmin, const double *kmax, int n_pages,
                    double *ub, double *S)
{
    for (int j = 0; j < n_pages; ++j) {
        double group = 0.0;
        for (int g = 0; g < G; ++g) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) {
                double a = q[(size_t)g * d + c] * kmin[(size_t)j * d + c];
                double b = q[(size_t)g * d + c] * kmax[(size_t)j * d + c];
                acc += a > b ? a : b;
            }
            acc *= scale;
            if (ub) ub[(size_t)g * n_pages + j] = acc;
            group += acc;
        }
        if (S) S[j] = group;
    }
}

/* ---------------------------------------------------------------------------------------
 * §2.A Gaussian page model of the token scores s = scale * q.k for one query:
 *   m_{g,j} = scale * sum_c q_{g,c} mu_{j,c}
 *   v_{g,j} = scale^2 * sum_c q_{g,c}^2 sigma^2_{j,c}   (coordinates treated as independent)
 * m, v: [G][n_pages].
 * ------------------------------------------------------------------------------------- */
void ora_gauss_stats_head(const double *q, int G, int d, double scale,
                          const double *mean, const double *var, int n_pages,
                          double *m, double *v)
{
    for (int g = 0; g < G; ++g)
        for (int j = 0; j < n_pages; ++j) {
            double a = 0.0, b = 0.0;
            for (int c = 0; c < d; ++c) {
                double qc = q[(size_t)g * d + c];
                a += qc * mean[(size_t)j * d + c];
                b += qc * qc * var[(size_t)j * d + c];
            }
            m[(size_t)g * n_pages + j] = scale * a;
            v[(size_t)g * n_pages + j] = scale * scale * b;
        }
}

/* ---------------------------------------------------------------------------------------
 * §2.B.1 top-k pages: order pages by (S descending, page index ascending), keep the first
 * min(k, n) of them, emit them in ascending page order. Returns the count.
 * ------------------------------------------------------------------------------------- */
static const double *g_sort_keys;

static int cmp_score_desc(const void *pa, const void *pb)
{
    int a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    double sa = g_sort_keys[a], sb = g_sort_keys[b];
    if (sa > sb) return -1;
    if (sa < sb) return 1;
    return a < b ? -1 : (a > b);
}

static int cmp_int_asc(const void *pa, const void *pb)
{
    int a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return a < b ? -1 : (a > b);
}

int ora_topk(const double *S, int n, int k, int32_t *sel)
{
    if (n <= 0 || k <= 0)
        return 0;
    int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    for (int j = 0; j < n; ++j)
        order[j] = j;
    g_sort_keys = S;
    qsort(order, (size_t)n, sizeof(int32_t), cmp_score_desc);
    int cnt = k < n ? k : n;
    memcpy(sel, order, sizeof(int32_t) * (size_t)cnt);
    qsort(sel, (size_t)cnt, sizeof(int32_t), cmp_int_asc);
    free(order);
    return cnt;
}

/* ---------------------------------------------------------------------------------------
 * §2.B.2 Gaussian-aware threshold.
 * With X ~ N(a, b^2) the expected entmax mass of one token at threshold tau is
 *   E[(X - tau)_+^(1/(alpha-1))]
 * alpha = 2 (power 1):   (a - tau) Phi(u) + b phi(u),                       u = (a - tau)/b
 * alpha = 1.5 (power 2): ((a - tau)^2 + b^2) Phi(u) + (a - tau) b phi(u)
 * b = 0: (a - tau)_+^(1/(alpha-1)).
 * ------------------------------------------------------------------------------------- */
static double std_normal_cdf(double u) { return 0.5 * erfc(-u / sqrt(2.0)); }
static double std_normal_pdf(double u) { return exp(-0.5 * u * u) / sqrt(2.0 * M_PI); }

double ora_trunc_moment(double a, double b, double tau, double alpha)
{
    double r = a - tau;
    if (b <= 0.0) {
        if (r <= 0.0) return 0.0;
        return alpha == 2.0 ? r : r * r;
    }
    double u = r / b;
    double Phi = std_normal_cdf(u), phi = std_normal_pdf(u);
    if (alpha == 2.0)
        return r * Phi + b * phi;
    if (alpha == 1.5)
        return (r * r + b * b) * Phi + r * b * phi;
    return NAN;
}

/* F(tau) = sum_j n_j * E_j(tau), with a_j = (alpha-1) m_j and b_j = (alpha-1) sqrt(v_j):
 * the expected total entmax mass when page j's n_j token scores are iid N(m_j, v_j). */
double ora_gauss_F(const double *m, const double *v, const int32_t *cnt, int n_pages,
                   double alpha, double tau)
{
    double F = 0.0;
    for (int j = 0; j < n_pages; ++j) {
        double a = (alpha - 1.0) * m[j];
        double b = (alpha - 1.0) * sqrt(v[j] > 0.0 ? v[j] : 0.0);
        F += (double)cnt[j] * ora_trunc_moment(a, b, tau, alpha);
    }
    return F;
}

/* Solve F(tau-hat) = 1 by bisection. F is continuous and non-increasing, and strictly
 * decreasing wherever it is positive. Lower end: at tau = max_j a_j - 1 the page with the
 * largest a alone contributes n_j E[(X - tau)_+^p] >= (E[X] - tau)^p = 1 (Jensen), so F >= 1.
 * Upper end: max_j (a_j + 10 b_j), pushed up until F < 1. No pages: -inf. */
double ora_gauss_tau(const double *m, const double *v, const int32_t *cnt, int n_pages,
                     double alpha)
{
    if (n_pages <= 0)
        return -INFINITY;
    double amax = -INFINITY, hi = -INFINITY;
    for (int j = 0; j < n_pages; ++j) {
        double a = (alpha - 1.0) * m[j];
        double b = (alpha - 1.0) * sqrt(v[j] > 0.0 ? v[j] : 0.0);
        if (a > amax) amax = a;
        if (a + 10.0 * b > hi) hi = a + 10.0 * b;
    }
    double lo = amax - 1.0;
    for (int it = 0; it < 200 && ora_gauss_F(m, v, cnt, n_pages, alpha, lo) < 1.0; ++it)
        lo -= 1.0 + (hi - lo);
    for (int it = 0; it < 200 && ora_gauss_F(m, v, cnt, n_pages, alpha, hi) >= 1.0; ++it)
        hi += 1.0 + (hi - lo);
    for (int it = 0; it < 500; ++it) {
        double mid = 0.5 * (lo + hi);
        if (hi - lo <= 1e-13 * (fabs(mid) > 1.0 ? fabs(mid) : 1.0))
            break;
        if (ora_gauss_F(m, v, cnt, n_pages, alpha, mid) >= 1.0)
            lo = mid;
        else
            hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* Keep page j iff some query g of the group has (alpha-1) * UB_{g,j} > tau_hat_g - delta.
 * ub: [G][n_pages]; emits ascending page indices, returns the count. */
int ora_gauss_select(const double *ub, const double *tau_hat, int G, int n_pages,
                     double alpha, double delta, int32_t *sel)
{
    int cnt = 0;
    for (int j = 0; j < n_pages; ++j) {
        int keep = 0;
        for (int g = 0; g < G; ++g)
            if ((alpha - 1.0) * ub[(size_t)g * n_pages + j] > tau_hat[g] - delta)
                keep = 1;
        if (keep)
            sel[cnt++] = j;
    }
    return cnt;
}

/* Second reading of the "estimated maximum score" (§2.B.2): a page's n token scores are modelled
 * as n draws from N(m, v); the expected largest of n standard normal draws is at most
 * sqrt(2 ln n), so m + sqrt(2 ln n) sqrt(v) estimates the page maximum. The bounding-box bound
 * holds exactly, so the estimate is capped by it. One token: the estimate is m (v = 0). */
double ora_est_max(double ub, double m, double v, int n)
{
    const double z = n > 1 ? sqrt(2.0 * log((double)n)) : 0.0;
    const double e = m + z * sqrt(v > 0.0 ? v : 0.0);
    return e < ub ? e : ub;
}

/* Keep page j iff some query g has (alpha-1) * est_{g,j} > tau_hat_g - delta, with est the
 * capped Gaussian estimate above. ub, m, v: [G][n_pages]; cnt: the pages' token counts. */
int ora_gauss_select_est(const double *ub, const double *m, const double *v, const int32_t *cnt,
                         const double *tau_hat, int G, int n_pages, double alpha, double delta,
                         int32_t *sel)
{
    int kept = 0;
    for (int j = 0; j < n_pages; ++j) {
        int keep = 0;
        for (int g = 0; g < G; ++g) {
            const size_t i = (size_t)g * n_pages + j;
            if ((alpha - 1.0) * ora_est_max(ub[i], m[i], v[i], cnt[j]) > tau_hat[g] - delta)
                keep = 1;
        }
        if (keep)
            sel[kept++] = j;
    }
    return kept;
}

/* ---------------------------------------------------------------------------------------
 * §2.C exact alpha-entmax threshold by sorting, for alpha in {1.5, 2}, in the z domain:
 *   sum_i [z_i - tau]_+^(1/(alpha-1)) = 1.
 * Sort z descending. For a candidate support of the top k:
 *   alpha = 2:   tau(k) = (sum_{i<=k} z_(i) - 1) / k
 *   alpha = 1.5: sum_{i<=k} (z_(i) - tau)^2 = 1  =>  tau(k) = M_k - sqrt((1 - k s_k) / k),
 *                M_k the mean and s_k the population variance of the top k (needs 1 - k s_k >= 0).
 * The support size is the largest k with tau(k) <= z_(k); tau = tau(k) there.
 * (Sparsemax: Martins & Astudillo 2016; 1.5-entmax: Peters, Niculae & Martins 2019.)
 * Returns -inf for n = 0.
 * ------------------------------------------------------------------------------------- */
static int cmp_double_desc(const void *pa, const void *pb)
{
    double a = *(const double *)pa, b = *(const double *)pb;
    return a > b ? -1 : (a < b);
}

double ora_entmax_tau(const double *z, int n, double alpha)
{
    if (n <= 0)
        return -INFINITY;
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    memcpy(s, z, sizeof(double) * (size_t)n);
    qsort(s, (size_t)n, sizeof(double), cmp_double_desc);
    double tau = NAN, sum = 0.0, mean = 0.0, m2 = 0.0;
    for (int k = 1; k <= n; ++k) {
        double x = s[k - 1];
        double tk;
        if (alpha == 2.0) {
            sum += x;
            tk = (sum - 1.0) / k;
        } else {
            /* running mean and sum of squared deviations (Welford) */
            double dlt = x - mean;
            mean += dlt / k;
            m2 += dlt * (x - mean);
            double disc = (1.0 - m2) / k; /* (1 - k * s_k) / k with s_k = m2 / k */
            if (disc < 0.0)
                continue;
            tk = mean - sqrt(disc);
        }
        if (tk <= x)
            tau = tk;
    }
    free(s);
    return tau;
}

/* ---------------------------------------------------------------------------------------
 * §2.C attention for the G query heads of one KV head over a list of token rows (cache block,
 * position), visited in list order.
 *   s_i = scale * q_g . k_i
 *   softmax:  p_i = exp(s_i - max s) / sum,       stat = log sum_i exp(s_i)
 *   entmax:   z_i = (alpha-1) s_i, tau exact,     p_i = [z_i - tau]_+^(1/(alpha-1)), stat = tau
 *   o_g = sum_i p_i v_i
 * q: [G][d]; out: [G][d]; stat: [G]; weights (optional): [G][n_tok] in list order.
 * ------------------------------------------------------------------------------------- */
static void attend_rows(const void *k_cache, const void *v_cache, int dtype, int H_kv, int P,
                        int d, const int *blk, const int *pos, int n_tok, int h, const double *q,
                        int G, double scale, int mode, double *out, double *stat, double *weights)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)(n_tok > 0 ? n_tok : 1));
    double *p = (double *)malloc(sizeof(double) * (size_t)(n_tok > 0 ? n_tok : 1));
    double alpha = mode == ORA_ENTMAX15 ? 1.5 : 2.0;
    for (int g = 0; g < G; ++g) {
        const double *qg = q + (size_t)g * d;
        double *og = out + (size_t)g * d;
        for (int c = 0; c < d; ++c)
            og[c] = 0.0;
        if (n_tok == 0) {
            stat[g] = -INFINITY;
            continue;
        }
        for (int i = 0; i < n_tok; ++i) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += qg[c] * elem(k_cache, dtype, cache_off(blk[i], h, pos[i], c, H_kv, P, d));
            s[i] = scale * acc;
        }
        if (mode == ORA_SOFTMAX) {
            double mx = -INFINITY, l = 0.0;
            for (int i = 0; i < n_tok; ++i)
                if (s[i] > mx) mx = s[i];
            for (int i = 0; i < n_tok; ++i) {
                p[i] = exp(s[i] - mx);
                l += p[i];
            }
            for (int i = 0; i < n_tok; ++i)
                p[i] /= l;
            stat[g] = mx + log(l);
        } else {
            for (int i = 0; i < n_tok; ++i)
                s[i] *= alpha - 1.0; /* s now holds z */
            double tau = ora_entmax_tau(s, n_tok, alpha);
            for (int i = 0; i < n_tok; ++i) {
                double r = s[i] - tau;
                p[i] = r > 0.0 ? (alpha == 2.0 ? r : r * r) : 0.0;
            }
            stat[g] = tau;
        }
        for (int i = 0; i < n_tok; ++i) {
            if (weights) weights[(size_t)g * n_tok + i] = p[i];
            if (p[i] == 0.0) continue;
            for (int c = 0; c < d; ++c)
                og[c] += p[i] * elem(v_cache, dtype, cache_off(blk[i], h, pos[i], c, H_kv, P, d));
        }
    }
    free(s);
    free(p);
}

/* Attention over the selected pages of one sequence: tokens page by page in the order of `sel`
 * (ascending logical page index), then by position; only t < seq_len exist. Returns the token
 * count, or -1 when a selected page or its page-table entry is out of range. */
int ora_attend_head(const void *k_cache, const void *v_cache, int dtype, int num_blocks,
                    int H_kv, int P, int d, const int32_t *pt_row, int seq_len, int h,
                    const double *q, int G, double scale, int mode,
                    const int32_t *sel, int n_sel, double *out, double *stat, double *weights)
{
    int n_pages = pages_of(seq_len, P);
    int n_tok = 0;
    for (int i = 0; i < n_sel; ++i) {
        int j = sel[i];
        if (j < 0 || j >= n_pages || pt_row[j] < 0 || pt_row[j] >= num_blocks)
            return -1;
        n_tok += seq_len - j * P < P ? seq_len - j * P : P;
    }
    int *blk = (int *)malloc(sizeof(int) * (size_t)(n_tok > 0 ? n_tok : 1));
    int *pos = (int *)malloc(sizeof(int) * (size_t)(n_tok > 0 ? n_tok : 1));
    int t_all = 0;
    for (int i = 0; i < n_sel; ++i) {
        int j = sel[i];
        int n = seq_len - j * P < P ? seq_len - j * P : P;
        for (int t = 0; t < n; ++t) {
            blk[t_all] = pt_row[j];
            pos[t_all] = t;
            ++t_all;
        }
    }
    attend_rows(k_cache, v_cache, dtype, H_kv, P, d, blk, pos, n_tok, h, q, G, scale, mode, out,
                stat, weights);
    free(blk);
    free(pos);
    return n_tok;
}

/* ---------------------------------------------------------------------------------------
 * Token-level selection inside the selected pages, one selection per KV head (JSSA, "Joint
 * Subspace Sparse Attention for efficient long-context decoding", abstract on ai.info:
 * token-granular selection and an attention kernel indexed into the standard GQA cache
 * layout, with distinct selections per KV head). Readings:
 *   - a candidate token's score for KV head h is the sum over the G query heads of the group of
 *     scale * q_g . k, taken in the full key space (JSSA scores in a low-dimensional subspace
 *     fitted to data; with no data the subspace is the whole space, the full-rank limit);
 *   - candidates are the valid tokens of the selected pages, numbered in visiting order (page
 *     order of `sel`, then position); the T best by (score descending, number ascending) are
 *     kept and emitted in candidate order as (logical page, position) pairs.
 * Returns min(T, candidates), or -1 when a selected page or its page-table entry is out of
 * range.
 * ------------------------------------------------------------------------------------- */
int ora_token_topk_head(const void *k_cache, int dtype, int num_blocks, int H_kv, int P, int d,
                        const int32_t *pt_row, int seq_len, int h, const double *q, int G,
                        double scale, const int32_t *sel, int n_sel, int T, int32_t *tok_page,
                        int32_t *tok_pos)
{
    int n_pages = pages_of(seq_len, P);
    int n_cand = 0;
    for (int i = 0; i < n_sel; ++i) {
        int j = sel[i];
        if (j < 0 || j >= n_pages || pt_row[j] < 0 || pt_row[j] >= num_blocks)
            return -1;
        n_cand += seq_len - j * P < P ? seq_len - j * P : P;
    }
    if (n_cand == 0 || T <= 0)
        return 0;
    int32_t *cpage = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_cand);
    int32_t *cpos = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_cand);
    double *score = (double *)malloc(sizeof(double) * (size_t)n_cand);
    int32_t *kept = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_cand);
    int m = 0;
    for (int i = 0; i < n_sel; ++i) {
        int j = sel[i];
        int n = seq_len - j * P < P ? seq_len - j * P : P;
        for (int t = 0; t < n; ++t) {
            double acc = 0.0;
            for (int g = 0; g < G; ++g) {
                double sg = 0.0;
                for (int c = 0; c < d; ++c)
                    sg += q[(size_t)g * d + c] * elem(k_cache, dtype, cache_off(pt_row[j], h, t, c, H_kv, P, d));
                acc += scale * sg;
            }
            cpage[m] = j;
            cpos[m] = t;
            score[m] = acc;
            ++m;
        }
    }
    int cnt = ora_topk(score, n_cand, T, kept);  /* candidate numbers, ascending */
    for (int i = 0; i < cnt; ++i) {
        tok_page[i] = cpage[kept[i]];
        tok_pos[i] = cpos[kept[i]];
    }
    free(cpage);
    free(cpos);
    free(score);
    free(kept);
    return cnt;
}

/* Attention of the G queries over an explicit list of (logical page, position) tokens of one
 * sequence, read in place through the page table: the indexed attention of the token-level
 * selection above, with the arithmetic of ora_attend_head. Returns the token count, or -1 when a
 * page, a position or a page-table entry is out of range. */
int ora_attend_tokens_head(const void *k_cache, const void *v_cache, int dtype, int num_blocks,
                           int H_kv, int P, int d, const int32_t *pt_row, int seq_len, int h,
                           const double *q, int G, double scale, int mode,
                           const int32_t *tok_page, const int32_t *tok_pos, int n_tok,
                           double *out, double *stat)
{
    int n_pages = pages_of(seq_len, P);
    int *blk = (int *)malloc(sizeof(int) * (size_t)(n_tok > 0 ? n_tok : 1));
    int *pos = (int *)malloc(sizeof(int) * (size_t)(n_tok > 0 ? n_tok : 1));
    for (int i = 0; i < n_tok; ++i) {
        int j = tok_page[i], t = tok_pos[i];
        if (j < 0 || j >= n_pages || pt_row[j] < 0 || pt_row[j] >= num_blocks || t < 0 ||
            t >= P || j * P + t >= seq_len) {
            free(blk);
            free(pos);
            return -1;
        }
        blk[i] = pt_row[j];
        pos[i] = t;
    }
    attend_rows(k_cache, v_cache, dtype, H_kv, P, d, blk, pos, n_tok, h, q, G, scale, mode, out,
                stat, NULL);
    free(blk);
    free(pos);
    return n_tok;
}

/*
 * Moment-corrected sparse softmax ("MomentKV", technical summary on gist.science,
 * Methodology §1, §2 and §4), read for a paged cache that keeps every token but skips the
 * pages a decode step did not select:
 *   - the evicted set E of the step is every valid token of the sequence outside the selected
 *     pages; its statistics are taken from E's rows directly: n_e, the key mean kbar, the value
 *     mean vbar and the centred value-key cross moment St = sum_E (v - vbar)(k - kbar)^T;
 *   - first-order estimate of the softmax output over E (logits s = scale q.k expanded around
 *     scale q.kbar, §2): fE = vbar + (scale / n_e) St q -- the summary's 1/(n_e sqrt(d)) is this
 *     factor at scale = 1/sqrt(d);
 *   - Jensen lower bound on E's partition sum (§4): ZE = n_e exp(scale q.kbar);
 *   - with fR, ZR the plain softmax output and partition sum over the selected pages:
 *     out = wR fR + (1 - wR) fE, wR = ZR / (ZR + ZE), stat = log(ZR + ZE).
 * Returns n_e, or -1 when a selected page or page-table entry is out of range.
 */
int ora_moment_corrected_head(const void *k_cache, const void *v_cache, int dtype, int num_blocks,
                              int H_kv, int P, int d, const int32_t *pt_row, int seq_len, int h,
                              const double *q, int G, double scale, const int32_t *sel, int n_sel,
                              double *out, double *stat)
{
    if (ora_attend_head(k_cache, v_cache, dtype, num_blocks, H_kv, P, d, pt_row, seq_len, h, q, G,
                        scale, ORA_SOFTMAX, sel, n_sel, out, stat, NULL) < 0)
        return -1;
    const int n_pages = pages_of(seq_len, P);
    char *kept = (char *)calloc((size_t)(n_pages > 0 ? n_pages : 1), 1);
    for (int i = 0; i < n_sel; ++i)
        kept[sel[i]] = 1;
    int n_e = 0;
    for (int j = 0; j < n_pages; ++j) {
        if (kept[j]) continue;
        if (pt_row[j] < 0 || pt_row[j] >= num_blocks) {
            free(kept);
            return -1;
        }
        n_e += seq_len - j * P < P ? seq_len - j * P : P;
    }
    if (n_e == 0) {
        free(kept);
        return 0;
    }
    double *kbar = (double *)calloc((size_t)d, sizeof(double));
    double *vbar = (double *)calloc((size_t)d, sizeof(double));
    double *St = (double *)calloc((size_t)d * d, sizeof(double));
    double *dv = (double *)malloc(sizeof(double) * (size_t)d);
    double *dk = (double *)malloc(sizeof(double) * (size_t)d);
    double *fE = (double *)malloc(sizeof(double) * (size_t)d);
    for (int j = 0; j < n_pages; ++j) {
        if (kept[j]) continue;
        const int n = seq_len - j * P < P ? seq_len - j * P : P;
        for (int t = 0; t < n; ++t)
            for (int c = 0; c < d; ++c) {
                kbar[c] += elem(k_cache, dtype, cache_off(pt_row[j], h, t, c, H_kv, P, d));
                vbar[c] += elem(v_cache, dtype, cache_off(pt_row[j], h, t, c, H_kv, P, d));
            }
    }
    for (int c = 0; c < d; ++c) {
        kbar[c] /= n_e;
        vbar[c] /= n_e;
    }
    for (int j = 0; j < n_pages; ++j) {
        if (kept[j]) continue;
        const int n = seq_len - j * P < P ? seq_len - j * P : P;
        for (int t = 0; t < n; ++t) {
            for (int c = 0; c < d; ++c) {
                dk[c] = elem(k_cache, dtype, cache_off(pt_row[j], h, t, c, H_kv, P, d)) - kbar[c];
                dv[c] = elem(v_cache, dtype, cache_off(pt_row[j], h, t, c, H_kv, P, d)) - vbar[c];
            }
            for (int a = 0; a < d; ++a)
                for (int c = 0; c < d; ++c)
                    St[(size_t)a * d + c] += dv[a] * dk[c];
        }
    }
    for (int g = 0; g < G; ++g) {
        const double *qg = q + (size_t)g * d;
        double *og = out + (size_t)g * d;
        double sbar = 0.0;
        for (int c = 0; c < d; ++c)
            sbar += qg[c] * kbar[c];
        sbar *= scale;
        for (int a = 0; a < d; ++a) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += St[(size_t)a * d + c] * qg[c];
            fE[a] = vbar[a] + scale / n_e * acc;
        }
        const double logZR = stat[g];  /* -inf when no token is selected */
        const double logZE = log((double)n_e) + sbar;
        const double mx = logZR > logZE ? logZR : logZE;
        const double zr = exp(logZR - mx), ze = exp(logZE - mx);
        const double wR = zr / (zr + ze);
        for (int a = 0; a < d; ++a)
            og[a] = wR * og[a] + (1.0 - wR) * fE[a];
        stat[g] = mx + log(zr + ze);
    }
    free(kept);
    free(kbar);
    free(vbar);
    free(St);
    free(dv);
    free(dk);
    free(fE);
    return n_e;
}

/* Moment sums of one (sequence, KV head) over the valid tokens of the listed logical pages
 * (MomentKV technical summary, Methodology §1: count, key sum, value sum and value-key
 * outer-product sum): n, sk [d], sv [d], S [d][d] with S[a][c] = sum v_a k_c.
 * Returns n, or -1 when a page or page-table entry is out of range. */
int ora_moment_sums_head(const void *k_cache, const void *v_cache, int dtype, int num_blocks,
                         int H_kv, int P, int d, const int32_t *pt_row, int seq_len, int h,
                         const int32_t *pages, int n_list, double *sk, double *sv, double *S)
{
    const int n_pages = pages_of(seq_len, P);
    for (int c = 0; c < d; ++c)
        sk[c] = sv[c] = 0.0;
    for (size_t i = 0; i < (size_t)d * d; ++i)
        S[i] = 0.0;
    int n = 0;
    for (int i = 0; i < n_list; ++i) {
        const int j = pages[i];
        if (j < 0 || j >= n_pages || pt_row[j] < 0 || pt_row[j] >= num_blocks)
            return -1;
        const int cnt = seq_len - j * P < P ? seq_len - j * P : P;
        for (int t = 0; t < cnt; ++t) {
            for (int a = 0; a < d; ++a) {
                const double va = elem(v_cache, dtype, cache_off(pt_row[j], h, t, a, H_kv, P, d));
                sv[a] += va;
                for (int c = 0; c < d; ++c)
                    S[(size_t)a * d + c] += va * elem(k_cache, dtype, cache_off(pt_row[j], h, t, c, H_kv, P, d));
            }
            for (int c = 0; c < d; ++c)
                sk[c] += elem(k_cache, dtype, cache_off(pt_row[j], h, t, c, H_kv, P, d));
            ++n;
        }
    }
    return n;
}

/* ---------------------------------------------------------------------------------------
 * How much of the full-cache attention a page selection keeps, per query g of KV head h
 * (EntmaxKV summary §3: attending over a subset of the tokens moves the output by at most
 * 2 B delta, delta the full-cache weight outside the subset; §3-§4: whether the kept pages
 * hold the support of the full-cache entmax). Over every valid token i of the sequence:
 *   p_i   the full-cache weight. With stat == NULL it is the weight of the attention over all
 *         pages (attend_rows over every token, in page order). With stat given ([G], the
 *         full-cache log-partition for softmax, the threshold tau for entmax) it is the
 *         weight that statistic defines: exp(s_i - stat_g), or [z_i - stat_g]_+^(1/(alpha-1))
 *         with z = (alpha-1) s.
 *   dropped[g]  sum of p_i over the tokens of pages outside `sel` (delta)
 *   n_sup[g]    entmax: tokens with p_i > 0 (the support); softmax: every valid token
 *   n_kept[g]   those of the n_sup[g] tokens that lie in a page of `sel`
 * Returns the sequence's token count, or -1 when a selected page or a page-table entry is out
 * of range.
 * ------------------------------------------------------------------------------------- */
int ora_selection_quality_head(const void *k_cache, const void *v_cache, int dtype,
                               int num_blocks, int H_kv, int P, int d, const int32_t *pt_row,
                               int seq_len, int h, const double *q, int G, double scale,
                               int mode, const double *stat, const int32_t *sel, int n_sel,
                               double *dropped, int32_t *n_sup, int32_t *n_kept)
{
    int n_pages = pages_of(seq_len, P);
    for (int j = 0; j < n_pages; ++j)
        if (pt_row[j] < 0 || pt_row[j] >= num_blocks)
            return -1;
    char *kept = (char *)calloc((size_t)(n_pages > 0 ? n_pages : 1), 1);
    for (int i = 0; i < n_sel; ++i) {
        if (sel[i] < 0 || sel[i] >= n_pages) {
            free(kept);
            return -1;
        }
        kept[sel[i]] = 1;
    }
    int n_tok = seq_len > 0 ? seq_len : 0;
    size_t nb = (size_t)(n_tok > 0 ? n_tok : 1);
    int *blk = (int *)malloc(sizeof(int) * nb);
    int *pos = (int *)malloc(sizeof(int) * nb);
    char *in_sel = (char *)malloc(nb);
    for (int i = 0; i < n_tok; ++i) {
        blk[i] = pt_row[i / P];
        pos[i] = i % P;
        in_sel[i] = kept[i / P];
    }
    double *w = (double *)malloc(sizeof(double) * nb * (size_t)G);
    if (!stat) {
        double *out = (double *)malloc(sizeof(double) * (size_t)G * d);
        double *st = (double *)malloc(sizeof(double) * (size_t)G);
        attend_rows(k_cache, v_cache, dtype, H_kv, P, d, blk, pos, n_tok, h, q, G, scale, mode,
                    out, st, w);
        free(out);
        free(st);
    } else {
        double alpha = mode == ORA_ENTMAX15 ? 1.5 : 2.0;
        for (int g = 0; g < G; ++g)
            for (int i = 0; i < n_tok; ++i) {
                double acc = 0.0;
                for (int c = 0; c < d; ++c)
                    acc += q[(size_t)g * d + c] *
                           elem(k_cache, dtype, cache_off(blk[i], h, pos[i], c, H_kv, P, d));
                double s = scale * acc, p;
                if (mode == ORA_SOFTMAX) {
                    p = exp(s - stat[g]);
                } else {
                    double r = (alpha - 1.0) * s - stat[g];
                    p = r > 0.0 ? (alpha == 2.0 ? r : r * r) : 0.0;
                }
                w[(size_t)g * n_tok + i] = p;
            }
    }
    for (int g = 0; g < G; ++g) {
        double dsum = 0.0;
        int ns = 0, nk = 0;
        for (int i = 0; i < n_tok; ++i) {
            double p = w[(size_t)g * n_tok + i];
            if (!in_sel[i]) dsum += p;
            int member = mode == ORA_SOFTMAX ? 1 : p > 0.0;
            ns += member;
            nk += member && in_sel[i];
        }
        dropped[g] = dsum;
        n_sup[g] = ns;
        n_kept[g] = nk;
    }
    free(w);
    free(in_sel);
    free(pos);
    free(blk);
    free(kept);
    return n_tok;
}
