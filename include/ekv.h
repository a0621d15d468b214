/*
 * ekv.h -- C ABI of libekv: query-aware sparse decode attention over a paged KV cache on
 * NVIDIA B200 (sm_100a).
 *
 * The method ("EntmaxKV: support-aware decoding for alpha-entmax attention", technical
 * summary on gist.science): the KV cache is split into pages (§2); per-page key metadata --
 * a coordinate-wise kmin/kmax bounding box and the key mean/variance -- is kept up to date as
 * pages fill (§2.A); each decode step scores every page with a query-aware bound before any
 * key or value is loaded (§2.A), selects candidate pages either as a fixed top-k budget
 * (§2.B.1) or as the pages whose estimated maximum score clears a Gaussian-estimated entmax
 * threshold tau-hat less a margin Delta (§2.B.2), and runs exact alpha-entmax (or softmax)
 * attention over only those pages (§2.C).
 *
 * Conventions shared by every call
 *  - All pointers are caller-owned DEVICE memory, except `c` itself (a host struct) and the
 *    host outputs of ekv_device_status. The library never allocates or frees memory.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and returns an ekv_status. Only ekv_device_status synchronises.
 *  - Host-side validation failures return before any launch and leave every output
 *    untouched. Supported shapes: head_dim d in {64, 128}; page size P in {16, 32, 64};
 *    K/V/q/bbox dtype fp32 or bf16; num_q_heads a multiple of num_kv_heads with group size
 *    G = num_q_heads / num_kv_heads in {1, 2, 4, 8}.
 *  - Device-side bad input (a page-table entry outside [0, num_blocks), a sequence length
 *    outside [0, max_pages * P], a selected page outside the sequence, ...) never traps:
 *    the offending page is skipped and an EKV_DEV_* bit is OR-ed into *c->dev_status.
 *    Read it with ekv_device_status.
 *  - Logits are s = scale * q.k. The alpha-entmax weights are p_i = [z_i - tau]_+^(1/(alpha-1))
 *    with z = (alpha - 1) s and sum_i p_i = 1 (alpha = 1.5 or alpha = 2, sparsemax).
 *  - Page j of sequence b holds tokens j*P .. j*P+P-1; only tokens t < seq_lens[b] exist, so
 *    the last page of a sequence may be partly filled. Pages j >= ceil(seq_lens[b] / P) do
 *    not exist.
 */
#ifndef EKV_H
#define EKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EKV_OK = 0,
    EKV_ERR_INVALID_ARG = 1, /* a null pointer, a negative size, a size mismatch         */
    EKV_ERR_UNSUPPORTED = 2, /* a shape / dtype / mode outside the supported set          */
    EKV_ERR_WORKSPACE = 3,   /* workspace smaller than ekv_decode_workspace_bytes()        */
    EKV_ERR_CUDA = 4,        /* a CUDA launch or copy failed                              */
    EKV_ERR_DEVICE = 5       /* ekv_device_status: a kernel flagged bad input             */
} ekv_status;

typedef enum { EKV_F32 = 0, EKV_BF16 = 1 } ekv_dtype;

/* attention over the selected pages (§2.C); alpha = 1, 1.5, 2 */
typedef enum { EKV_SOFTMAX = 0, EKV_ENTMAX15 = 1, EKV_SPARSEMAX = 2 } ekv_attn;

/* candidate selection policy (§2.B) */
typedef enum { EKV_SEL_TOPK = 0, EKV_SEL_GAUSS = 1, EKV_SEL_GAUSS_MAX = 2 } ekv_policy;

/* bits OR-ed into *dev_status by kernels that meet bad input */
#define EKV_DEV_BAD_BLOCK 0x1u    /* page-table entry outside [0, num_blocks)            */
#define EKV_DEV_BAD_LEN 0x2u      /* seq_lens[b] outside [0, max_pages * P]               */
#define EKV_DEV_BAD_SEL 0x4u      /* selected page outside [0, ceil(seq_len / P))         */
#define EKV_DEV_SEL_OVERFLOW 0x8u /* Gaussian policy kept more than max_sel pages         */
#define EKV_DEV_BAD_RANGE 0x10u   /* meta update range outside [0, seq_len] or > max_new   */
#define EKV_DEV_TIMEOUT 0x20u     /* a bounded on-chip wait gave up (the call's outputs are
                                     incomplete); not expected in normal operation          */

/*
 * The paged cache and its metadata (§2, §2.A). Plain data; every pointer is device memory.
 *   k_cache, v_cache  [num_blocks][H_kv][P][d] in `dtype`: one (block, head) is P*d
 *                     contiguous elements, so a page of one KV head is one contiguous span.
 *   meta_bbox         [num_blocks][H_kv][2][d] in `dtype`: row 0 kmin, row 1 kmax of the
 *                     page's valid keys (exact: min/max of stored values).
 *   meta_mom          [num_blocks][H_kv][2][d] fp32: row 0 mean, row 1 population variance of
 *                     the page's valid keys. NULL is allowed unless a Gaussian policy is used.
 *   page_table        [batch][max_pages] int32: logical page j of sequence b is block
 *                     page_table[b * max_pages + j].
 *   seq_lens          [batch] int32: tokens in each sequence.
 *   dev_status        one uint32 word of device memory; kernels OR EKV_DEV_* bits into it.
 */
typedef struct {
    int32_t dtype;        /* ekv_dtype of K, V, q and meta_bbox       */
    int32_t head_dim;     /* d                                        */
    int32_t page_size;    /* P                                        */
    int32_t num_kv_heads; /* H_kv                                     */
    int32_t num_blocks;   /* physical blocks in the pool              */
    int32_t batch;        /* B                                        */
    int32_t max_pages;    /* row length of page_table                 */
    int32_t reserved;     /* must be 0                                */
    void *k_cache;
    void *v_cache;
    void *meta_bbox;
    float *meta_mom;
    const int32_t *page_table;
    const int32_t *seq_lens;
    uint32_t *dev_status;
} ekv_cache;

/*
 * §2.A "metadata kept up to date as pages fill": recompute kmin/kmax (and, when meta_mom is
 * not NULL, mean and population variance) of every page touched by the token range
 * [new_start[b], new_start[b] + new_count[b]) of each sequence b, from all of that page's
 * valid tokens (t < seq_lens[b]; seq_lens must already count the new tokens).
 *   new_start, new_count  [batch] int32 device arrays (they stay on the device so a decode
 *                         loop never synchronises). new_count[b] = 0 touches nothing.
 *   max_new               host upper bound on every new_count[b]; sizes the launch. A range
 *                         longer than max_new, or outside [0, seq_lens[b]], is clamped and
 *                         flagged EKV_DEV_BAD_RANGE.
 * Prefill: new_start = 0, new_count = seq_lens, max_new = max(seq_lens).
 * c->k_cache must be 16-byte aligned (EKV_ERR_INVALID_ARG otherwise).
 */
ekv_status ekv_page_meta_update(const ekv_cache *c, const int32_t *new_start,
                                const int32_t *new_count, int32_t max_new, void *stream);

/*
 * §2.A query-aware page scores, computed from the metadata only.
 *   q       [batch][num_q_heads][d] in c->dtype; query head hq belongs to KV head hq / G.
 *   scale   logit scale (> 0): s = scale * q.k.
 *   policy  EKV_SEL_TOPK: scores is [batch][H_kv][max_pages] fp32 and holds the group bound
 *             S_j = sum_{g in group} UB_{g,j},  UB_{g,j} = scale * sum_c max(q_gc kmin_jc, q_gc kmax_jc).
 *           EKV_SEL_GAUSS, EKV_SEL_GAUSS_MAX: scores is [batch][num_q_heads][3][max_pages] fp32 and holds, per
 *             query, UB_{g,j}, m_{g,j} = scale * q_g.mean_j and
 *             v_{g,j} = scale^2 * sum_c q_gc^2 var_jc (needs c->meta_mom).
 * Entries for pages j >= ceil(seq_lens[b] / P) are not written. A page whose page-table entry
 * is out of range scores -inf (and m = v = 0) and is flagged.
 * c->meta_bbox (and c->meta_mom for the Gaussian policies) must be 16-byte aligned: metadata rows are
 * read with 16-byte vector loads (EKV_ERR_INVALID_ARG otherwise).
 */
ekv_status ekv_score_pages(const ekv_cache *c, const void *q, int32_t num_q_heads, float scale,
                           int32_t policy, float *scores, void *stream);

/*
 * §2.A both steps of a decode step's start in one call: ekv_page_meta_update(c, new_start,
 * new_count, max_new) followed by ekv_score_pages(c, q, num_q_heads, scale, policy, scores), with
 * the results of the two calls bit for bit (metadata, scores, device status bits). Under
 * EKV_SEL_TOPK with max_new <= 2 P and few (sequence, KV head) pairs (2 * batch * H_kv at most a
 * sixteenth of the scan's persistent grid), one kernel does both: leading blocks rebuild the
 * appended pages' metadata and score the 8-page groups holding them while the rest of the grid
 * scans every other group. Otherwise the two kernels run in turn. max_new = 0 is
 * ekv_score_pages alone.
 * Arguments, layouts, alignment and errors: those of the two calls.
 */
ekv_status ekv_refresh_score_pages(const ekv_cache *c, const int32_t *new_start,
                                   const int32_t *new_count, int32_t max_new, const void *q,
                                   int32_t num_q_heads, float scale, int32_t policy,
                                   float *scores, void *stream);

/*
 * §2.B candidate selection, per (sequence, KV head).
 *   EKV_SEL_TOPK (§2.B.1): the min(topk, n_pages) pages with the largest S_j; equal scores go
 *     to the lower page index. alpha, delta, tau_hat are ignored (tau_hat may be NULL).
 *     Requires max_sel >= min(topk, max_pages).
 *   EKV_SEL_GAUSS (§2.B.2): per query g, tau_hat_g solves
 *       sum_j n_j E[((alpha-1) s - tau)_+^(1/(alpha-1))] = 1,  s ~ N(m_{g,j}, v_{g,j}),
 *     n_j the valid tokens of page j (alpha in {1.5, 2}); page j is kept iff some query g of
 *     the group has (alpha-1) * UB_{g,j} > tau_hat_g - delta. tau_hat: [batch][num_q_heads]
 *     fp32 output (-inf for an empty sequence). More than max_sel kept pages: the first
 *     max_sel (ascending) are emitted, sel_count holds max_sel, EKV_DEV_SEL_OVERFLOW is set.
 *   EKV_SEL_GAUSS_MAX: the same tau_hat, with the second reading of §2.B.2's "estimated
 *     maximum score": page j is kept iff some query g has (alpha-1) * est_{g,j} >
 *     tau_hat_g - delta, est = min(UB_{g,j}, m_{g,j} + sqrt(2 ln n_j) * sqrt(v_{g,j})) -- the
 *     Gaussian estimate of the page's largest score, capped by the bound (fp64 decision).
 *   scores     as written by ekv_score_pages with the same policy; 16-byte aligned (rows are
 *              read as float4), else EKV_ERR_INVALID_ARG.
 *   sel_idx    [batch][H_kv][max_sel] int32 output: logical page indices, ascending, then -1.
 *   sel_count  [batch][H_kv] int32 output.
 */
ekv_status ekv_select_pages(const ekv_cache *c, int32_t num_q_heads, int32_t policy,
                            int32_t topk, float alpha, float delta, const float *scores,
                            int32_t *sel_idx, int32_t *sel_count, int32_t max_sel,
                            float *tau_hat, void *stream);

/*
 * §2.A and §2.B.1 in one call: the top-k page scores of ekv_score_pages (policy EKV_SEL_TOPK)
 * and the selection of ekv_select_pages, with the same results bit for bit. One
 * thread-block cluster per (sequence, KV head) scans the pair's metadata and selects from the
 * scores in its shared memory, so no kernel waits for the whole grid in between.
 *   scores     [batch][H_kv][max_pages] fp32 output, 16-byte aligned; may be NULL when every
 *              (sequence, KV head) fits the cluster kernel (at most 16 CTAs of 8192 pages),
 *              which is then the only path. A geometry beyond that runs the two standalone
 *              kernels, which pass the scores through `scores` (NULL: EKV_ERR_INVALID_ARG).
 *   sel_idx, sel_count, max_sel, topk  as in ekv_select_pages (max_sel >= min(topk, max_pages)).
 * c->meta_bbox must be 16-byte aligned.
 */
ekv_status ekv_score_select_pages(const ekv_cache *c, const void *q, int32_t num_q_heads,
                                  float scale, int32_t topk, float *scores, int32_t *sel_idx,
                                  int32_t *sel_count, int32_t max_sel, void *stream);

/*
 * §2.C attention over the selected pages only, read in place from the paged cache (no gather
 * copy). For each query head: s_i = scale * q.k_i over the valid tokens of the pages of its
 * KV head listed in sel_idx[b][h][0 .. min(sel_count, max_sel));
 *   EKV_SOFTMAX:   p = softmax(s);                        stat = log sum_i exp(s_i)
 *   EKV_ENTMAX15, EKV_SPARSEMAX: z = (alpha-1) s, exact tau with sum_i [z_i - tau]_+^(1/(alpha-1)) = 1,
 *                  p_i = [z_i - tau]_+^(1/(alpha-1));    stat = tau
 *   out[b][hq][:] = sum_i p_i v_i (fp32);  an empty selection gives out = 0, stat = -inf.
 *   q          [batch][num_q_heads][d] in c->dtype. q, c->k_cache and c->v_cache must be
 *              16-byte aligned (pages and query rows are moved with bulk copies), else
 *              EKV_ERR_INVALID_ARG.
 *   out        [batch][num_q_heads][d] fp32.   stat [batch][num_q_heads] fp32.
 *   ws         scratch of at least ekv_decode_workspace_bytes(c, num_q_heads, max_sel)
 *              bytes, 16-byte aligned (EKV_ERR_INVALID_ARG otherwise). Its contents need no
 *              initialisation: every word a call reads was written earlier in the same call.
 *              Calls that share one ws must not overlap on the GPU.
 */
ekv_status ekv_sparse_decode(const ekv_cache *c, const void *q, int32_t num_q_heads,
                             float scale, int32_t attn, const int32_t *sel_idx,
                             const int32_t *sel_count, int32_t max_sel, float *out, float *stat,
                             void *ws, size_t ws_bytes, void *stream);

/*
 * §2.B.1 and §2.C in one call: the top-k selection of ekv_select_pages (policy EKV_SEL_TOPK)
 * followed by ekv_sparse_decode on that selection. sel_idx and sel_count are outputs, equal to
 * those of ekv_select_pages with the same scores and topk; out and stat are those of
 * ekv_sparse_decode on them. The two kernels run back to back on `stream`, the decode launched
 * behind the selection (programmatic dependent launch), so the decode's thread-block clusters
 * are placed on the GPU while the selection runs.
 *   scores     as written by ekv_score_pages with EKV_SEL_TOPK; 16-byte aligned.
 *   topk, sel_idx, sel_count, max_sel   as in ekv_select_pages (max_sel >= min(topk,
 *              max_pages)).
 *   q, attn, scale, out, stat, ws, ws_bytes   as in ekv_sparse_decode (same alignment and
 *              workspace rules).
 */
ekv_status ekv_select_decode(const ekv_cache *c, const void *q, int32_t num_q_heads, float scale,
                             int32_t attn, int32_t topk, const float *scores, int32_t *sel_idx,
                             int32_t *sel_count, int32_t max_sel, float *out, float *stat,
                             void *ws, size_t ws_bytes, void *stream);

/* Scratch that ekv_sparse_decode_noalloc draws on: 16 MiB, held by every GPU that loads the
 * library until the process exits. */
#define EKV_NOALLOC_WS_BYTES (16u << 20)

/*
 * ekv_sparse_decode without a workspace argument. (The paper has no counterpart: this is a
 * library convenience.)
 * For callers that cannot allocate device memory -- an engine whose allocator has already
 * reserved all of HBM for the KV cache and its own pools, a latency-critical loop that must
 * not risk a synchronising cudaMalloc/cudaFree, a plug-in that is handed only its inputs and
 * outputs. The scratch is a fixed array inside the library; this call allocates nothing.
 *   Arguments and results are those of ekv_sparse_decode (minus ws / ws_bytes).
 *   A geometry whose ekv_decode_workspace_bytes() exceeds EKV_NOALLOC_WS_BYTES returns
 *   EKV_ERR_WORKSPACE and launches nothing.
 *   The first call on a device looks up the array's device address (once per device, with
 *   that device current); make that first call before any stream capture.
 *   Every call on a device shares the one array, which keeps the last call's contents
 *   (nothing in it has to start at zero): calls that overlap on the GPU -- concurrent streams,
 *   or several host threads -- race on it and must be serialised by the caller.
 */
ekv_status ekv_sparse_decode_noalloc(const ekv_cache *c, const void *q, int32_t num_q_heads,
                                     float scale, int32_t attn, const int32_t *sel_idx,
                                     const int32_t *sel_count, int32_t max_sel, float *out,
                                     float *stat, void *stream);

/* Scratch bytes ekv_sparse_decode needs for this cache geometry, num_q_heads and max_sel
 * (0 on invalid arguments). */
size_t ekv_decode_workspace_bytes(const ekv_cache *c, int32_t num_q_heads, int32_t max_sel);

/*
 * Moment correction of a softmax decode for the pages it skips (MomentKV technical summary,
 * gist.science, Methodology §1, §2, §4). (Not part of the EntmaxKV method: entmax gives the
 * skipped tokens exact zeros wherever the support is kept; this is the softmax remedy.)
 * The cache keeps every token and a decode step skips the pages it did not select: those tokens
 * form the evicted set E of that step.
 *
 * Running moments: per (sequence, KV head), sums over every token appended so far, one fp32
 * record of EKV_MOMENT_FLOATS(d) floats:
 *   [0] n (token count)   [1..3] 0   [4, 4+d) sum k   [4+d, 4+2d) sum v
 *   [4+2d, 4+2d+d*d) sum v k^T, row a = value coordinate, column c = key coordinate.
 * moments: [batch][H_kv] records, ekv_moment_bytes(c) bytes, zero-filled by the caller before
 * the first update.
 */
#define EKV_MOMENT_FLOATS(d) (4 + 2 * (d) + (d) * (d))

/* Bytes of the running-moment records of this cache geometry (0 on invalid arguments). */
size_t ekv_moment_bytes(const ekv_cache *c);

/*
 * Add the tokens [new_start[b], new_start[b] + new_count[b]) of every sequence b to its running
 * moments (every KV head). Each token must be added once: prefill with new_start = 0,
 * new_count = seq_lens, then each appended range. Arguments and range checks are those of
 * ekv_page_meta_update (a range outside [0, seq_lens[b]] or longer than max_new is clamped and
 * flagged EKV_DEV_BAD_RANGE; a bad page-table entry is skipped and flagged). Needs c->v_cache.
 */
ekv_status ekv_moment_update(const ekv_cache *c, float *moments, const int32_t *new_start,
                             const int32_t *new_count, int32_t max_new, void *stream);

/* Scratch bytes ekv_sparse_decode_moment needs (0 on invalid arguments). */
size_t ekv_moment_decode_workspace_bytes(const ekv_cache *c, int32_t num_q_heads,
                                         int32_t max_sel);

/*
 * ekv_sparse_decode with attn = EKV_SOFTMAX, then corrected for the skipped tokens E of each
 * (sequence, KV head), per query head (logits s = scale q.k):
 *   n_e = |E|, kbar, vbar = the mean key and value over E,
 *   fE = vbar + (scale / n_e) sum_E (v - vbar)(k - kbar)^T q     (first-order estimate of E's
 *        softmax output around the mean logit scale q.kbar),
 *   ZE = n_e exp(scale q.kbar)                                    (Jensen lower bound on E's
 *        partition sum),
 *   out = wR fR + (1 - wR) fE,  wR = ZR / (ZR + ZE),  stat = log(ZR + ZE),
 * with fR, log ZR the softmax output and stat over the selected pages. E's sums are the running
 * moments less the sums over the selected tokens, which this call re-reads. With nothing
 * skipped (n_e = 0) the result is the plain softmax. Arguments are those of
 * ekv_sparse_decode, plus `moments` (as kept by ekv_moment_update for exactly the tokens
 * [0, seq_lens[b]) of each sequence); ws holds at least
 * ekv_moment_decode_workspace_bytes(c, num_q_heads, max_sel) bytes under the same rules
 * (16-byte aligned, no initialisation needed).
 */
ekv_status ekv_sparse_decode_moment(const ekv_cache *c, const float *moments, const void *q,
                                    int32_t num_q_heads, float scale, const int32_t *sel_idx,
                                    const int32_t *sel_count, int32_t max_sel, float *out,
                                    float *stat, void *ws, size_t ws_bytes, void *stream);

/*
 * Token-level selection inside the selected pages, with attention indexed into the cache
 * (after the JSSA abstract on ai.info: token-granular selection, one selection per KV head,
 * attention on the standard GQA cache layout with no gather copy). Not part of EntmaxKV:
 * a finer granularity applied after its page selection.
 *   Candidates of (sequence b, KV head h): the valid tokens of the pages in
 *   sel_idx[b][h][0 .. sel_count), in that order and then by position. A candidate's score is
 *   the group sum sum_g scale * q_g . k over the G query heads of h (the full key space).
 *   The T best, ties to the earlier candidate, are kept in candidate order.
 */
#define EKV_MAX_TOKENS 32768 /* largest T */

/* Scratch bytes of ekv_select_tokens: one fp32 score per candidate slot,
 * batch * H_kv * max_sel * P * 4 (0 on invalid arguments). The scratch must be 16-byte
 * aligned and needs no initialisation. */
size_t ekv_token_workspace_bytes(const ekv_cache *c, int32_t max_sel);

/*
 *   tok_page, tok_pos  [batch][H_kv][T] int32 outputs: logical page and position of each kept
 *                      token, -1 padded.   tok_count [batch][H_kv] int32 output.
 *   T in [1, EKV_MAX_TOKENS] (EKV_ERR_UNSUPPORTED above, EKV_ERR_INVALID_ARG below);
 *   other arguments as in ekv_score_pages / ekv_sparse_decode.
 */
ekv_status ekv_select_tokens(const ekv_cache *c, const void *q, int32_t num_q_heads, float scale,
                             const int32_t *sel_idx, const int32_t *sel_count, int32_t max_sel,
                             int32_t T, int32_t *tok_page, int32_t *tok_pos, int32_t *tok_count,
                             void *ws, size_t ws_bytes, void *stream);

/*
 * Attention of every query head over the tokens ekv_select_tokens kept for its KV head, their K
 * and V rows read in place through the page table: softmax (stat = log-partition) or exact
 * alpha-entmax (stat = tau), as in ekv_sparse_decode; no kept token gives out = 0,
 * stat = -inf. A listed token outside its sequence is skipped and flagged EKV_DEV_BAD_SEL.
 */
ekv_status ekv_sparse_decode_tokens(const ekv_cache *c, const void *q, int32_t num_q_heads,
                                    float scale, int32_t attn, const int32_t *tok_page,
                                    const int32_t *tok_pos, const int32_t *tok_count, int32_t T,
                                    float *out, float *stat, void *stream);

/*
 * How much of the full-cache attention a page selection keeps: a diagnostic beside the decode
 * (EntmaxKV summary §3: attending over a subset moves the output by at most 2 B delta, delta the
 * full-cache weight outside the subset; §3-§4: support recovery). It reads every key of every
 * sequence, so it costs a full-cache pass. For each query head, over every valid token i:
 *   p_i        the full-cache weight that stat_full defines: softmax exp(s_i - stat),
 *              entmax [(alpha-1) s_i - stat]_+^(1/(alpha-1)), s = scale q.k_i.
 *   dropped    [batch][num_q_heads] fp64 output: sum of p_i over tokens of pages outside
 *              sel_idx[b][h][0 .. sel_count) -- delta.
 *   support    [batch][num_q_heads][2] int32 output: the support size (entmax: tokens with
 *              (alpha-1) s_i > stat; softmax: every valid token) and how many of those lie in
 *              the selected pages (support recall = support[1] / support[0]).
 *   stat_full  [batch][num_q_heads] fp32: the full-cache statistic, e.g. the stat of
 *              ekv_sparse_decode called with every page of every sequence selected.
 * Both outputs are overwritten (zeroed on `stream`, then accumulated). A bad page-table entry is
 * skipped and flagged EKV_DEV_BAD_BLOCK. Other arguments as in ekv_sparse_decode.
 */
ekv_status ekv_selection_quality(const ekv_cache *c, const void *q, int32_t num_q_heads,
                                 float scale, int32_t attn, const float *stat_full,
                                 const int32_t *sel_idx, const int32_t *sel_count,
                                 int32_t max_sel, double *dropped, int32_t *support,
                                 void *stream);

/* Synchronise `stream`, copy *c->dev_status to *bits (host pointer, may be NULL) and return
 * EKV_ERR_DEVICE if any bit is set, else EKV_OK (EKV_ERR_CUDA if the copy fails). */
ekv_status ekv_device_status(const ekv_cache *c, uint32_t *bits, void *stream);

/* Clear *c->dev_status (asynchronous). */
ekv_status ekv_clear_device_status(const ekv_cache *c, void *stream);

/*
 * Self-test of the device-side timeout reporting. (The paper has no counterpart: this is a
 * library diagnostic.) Every pipelined kernel bounds each of its waits with the global timer and
 * sets EKV_DEV_TIMEOUT in *c->dev_status when a limit (2 s) runs out, instead of hanging. This
 * call launches one thread that waits, with that same bounded wait, on a barrier nothing ever
 * completes, for limit_ns nanoseconds (at most 2e9; larger values: EKV_ERR_INVALID_ARG), then
 * sets EKV_DEV_TIMEOUT and returns. Asynchronous; read the bit with ekv_device_status.
 */
ekv_status ekv_wait_selftest(const ekv_cache *c, uint64_t limit_ns, void *stream);

/* A static, human-readable name for a status code. */
const char *ekv_status_str(ekv_status s);

#ifdef __cplusplus
}
#endif

#endif /* EKV_H */
