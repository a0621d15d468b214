// ekv_api.cu -- the C ABI of libekv (declared in include/ekv.h): host-side validation,
// workspace sizing and kernel dispatch. Every entry point is asynchronous on the caller's
// stream except ekv_device_status; nothing here allocates device memory.
#include <cmath>
#include <cstdlib>
#include <map>
#include <mutex>
#include <tuple>

#include "ekv_device.cuh"

namespace ekv {

cudaError_t launch_page_meta_update(const ekv_cache &c, const int32_t *new_start,
                                    const int32_t *new_count, int max_new, cudaStream_t st);
cudaError_t launch_score_pages(const ekv_cache &c, const void *q, int H_q, float scale,
                               int policy, float *scores, cudaStream_t st, bool pdl);
cudaError_t launch_refresh_score_pages(const ekv_cache &c, const int32_t *new_start,
                                       const int32_t *new_count, int max_new, const void *q,
                                       int H_q, float scale, int policy, float *scores,
                                       cudaStream_t st, bool pdl);
cudaError_t launch_select_pages(const ekv_cache &c, int H_q, int policy, int topk, float alpha,
                                float delta, const float *scores, int32_t *sel_idx,
                                int32_t *sel_count, int max_sel, float *tau_hat, cudaStream_t st,
                                bool pdl);
cudaError_t launch_sparse_decode(const ekv_cache &c, const void *q, int H_q, float scale,
                                 int attn, const int32_t *sel_idx, const int32_t *sel_count,
                                 int max_sel, float *out, float *stat, void *ws, cudaStream_t st,
                                 bool pdl);
size_t decode_workspace_bytes_all_modes(int batch, int H_q, int H, int D, int P, int dtype,
                                        int max_sel);
cudaError_t launch_moment_update(const ekv_cache &c, float *moments, const int32_t *new_start,
                                 const int32_t *new_count, int max_new, cudaStream_t st);
cudaError_t launch_moment_pass(const ekv_cache &c, const float *moments, const void *q, int H_q,
                               float scale, const int32_t *sel_idx, const int32_t *sel_count,
                               int max_sel, float *ret, float *out, float *stat, cudaStream_t st,
                               bool after_decode);
size_t moment_retained_bytes(int batch, int H_kv, int D, int G);
cudaError_t launch_token_scores(const ekv_cache &c, const void *q, int H_q, float scale,
                                const int32_t *sel_idx, const int32_t *sel_count, int max_sel,
                                float *tscores, cudaStream_t st);
cudaError_t launch_select_tokens(const ekv_cache &c, const float *tscores, const int32_t *sel_idx,
                                 const int32_t *sel_count, int max_sel, int T, int32_t *tok_page,
                                 int32_t *tok_pos, int32_t *tok_count, cudaStream_t st);
cudaError_t launch_token_attend(const ekv_cache &c, const void *q, int H_q, float scale, int attn,
                                const int32_t *tok_page, const int32_t *tok_pos,
                                const int32_t *tok_count, int T, float *out, float *stat,
                                cudaStream_t st);

cudaError_t launch_selection_quality(const ekv_cache &c, const void *q, int H_q, float scale,
                                     int attn, const float *stat_full, const int32_t *sel_idx,
                                     const int32_t *sel_count, int max_sel, double *dropped,
                                     int32_t *support, cudaStream_t st);

bool step_score_select_supported(const ekv_cache &c);
cudaError_t launch_wait_selftest(uint32_t *status, uint64_t limit_ns, cudaStream_t st);
cudaError_t launch_step_score_select(const ekv_cache &c, const void *q, int H_q, float scale,
                                     int topk, float *scores, int32_t *sel_idx, int32_t *sel_count,
                                     int max_sel, cudaStream_t st, bool pdl);

int persistent_grid_size(const void *kernel, int threads, size_t smem)
{
    static std::mutex mu;
    static std::map<std::tuple<const void *, int, size_t>, int> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    const auto key = std::make_tuple(kernel, dev, smem);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int sms = 148, per_sm = 1;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess
        || per_sm < 1)
        per_sm = 1;
    const int g = sms * per_sm;
    cache[key] = g;
    return g;
}

// Programmatic dependent launch between consecutive libekv kernels (EKV_PDL=0 turns it off).
bool use_pdl()
{
    static const bool on = [] {
        const char *e = std::getenv("EKV_PDL");
        return !(e && e[0] == '0');
    }();
    return on;
}

}  // namespace ekv

using namespace ekv;

static ekv_status check_cache(const ekv_cache *c, bool need_values)
{
    if (!c) return EKV_ERR_INVALID_ARG;
    if (c->dtype != EKV_F32 && c->dtype != EKV_BF16) return EKV_ERR_UNSUPPORTED;
    if (c->head_dim != 64 && c->head_dim != 128) return EKV_ERR_UNSUPPORTED;
    if (c->page_size != 16 && c->page_size != 32 && c->page_size != 64) return EKV_ERR_UNSUPPORTED;
    if (c->num_kv_heads < 1 || c->num_blocks < 1 || c->batch < 1 || c->max_pages < 1)
        return EKV_ERR_INVALID_ARG;
    if (c->batch > 8192) return EKV_ERR_UNSUPPORTED;
    if ((long long)c->max_pages * c->page_size > 0x7fffffffLL) return EKV_ERR_UNSUPPORTED;
    if ((long long)c->num_blocks * c->page_size > 0x7fffffffLL) return EKV_ERR_UNSUPPORTED;
    if (!c->k_cache || !c->meta_bbox || !c->page_table || !c->seq_lens || !c->dev_status)
        return EKV_ERR_INVALID_ARG;
    if (need_values && !c->v_cache) return EKV_ERR_INVALID_ARG;
    return EKV_OK;
}

static ekv_status check_heads(const ekv_cache *c, int32_t H_q)
{
    if (H_q < 1 || H_q % c->num_kv_heads != 0) return EKV_ERR_INVALID_ARG;
    const int G = H_q / c->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return EKV_ERR_UNSUPPORTED;
    return EKV_OK;
}

static ekv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? EKV_OK : EKV_ERR_CUDA; }

extern "C" {

ekv_status ekv_page_meta_update(const ekv_cache *c, const int32_t *new_start,
                                const int32_t *new_count, int32_t max_new, void *stream)
{
    ekv_status s = check_cache(c, false);
    if (s != EKV_OK) return s;
    if (!new_start || !new_count || max_new < 0) return EKV_ERR_INVALID_ARG;
    if ((uintptr_t)c->k_cache & 15u) return EKV_ERR_INVALID_ARG;  // rows are read with vector loads
    if ((long long)max_new > (long long)c->max_pages * c->page_size) return EKV_ERR_INVALID_ARG;
    return cuda_status(launch_page_meta_update(*c, new_start, new_count, max_new,
                                               static_cast<cudaStream_t>(stream)));
}

ekv_status ekv_score_pages(const ekv_cache *c, const void *q, int32_t num_q_heads, float scale,
                           int32_t policy, float *scores, void *stream)
{
    ekv_status s = check_cache(c, false);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    if (!q || !scores || !(scale > 0.0f) || !std::isfinite(scale)) return EKV_ERR_INVALID_ARG;
    if (policy != EKV_SEL_TOPK && policy != EKV_SEL_GAUSS && policy != EKV_SEL_GAUSS_MAX)
        return EKV_ERR_UNSUPPORTED;
    const bool gauss = policy != EKV_SEL_TOPK;
    if (gauss && !c->meta_mom) return EKV_ERR_INVALID_ARG;
    if ((uintptr_t)c->meta_bbox & 15u) return EKV_ERR_INVALID_ARG;
    if (gauss && ((uintptr_t)c->meta_mom & 15u)) return EKV_ERR_INVALID_ARG;
    return cuda_status(launch_score_pages(*c, q, num_q_heads, scale, policy, scores,
                                          static_cast<cudaStream_t>(stream), use_pdl()));
}

ekv_status ekv_refresh_score_pages(const ekv_cache *c, const int32_t *new_start,
                                   const int32_t *new_count, int32_t max_new, const void *q,
                                   int32_t num_q_heads, float scale, int32_t policy,
                                   float *scores, void *stream)
{
    ekv_status s = check_cache(c, false);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    // ekv_page_meta_update's checks
    if (!new_start || !new_count || max_new < 0) return EKV_ERR_INVALID_ARG;
    if ((uintptr_t)c->k_cache & 15u) return EKV_ERR_INVALID_ARG;
    if ((long long)max_new > (long long)c->max_pages * c->page_size) return EKV_ERR_INVALID_ARG;
    // ekv_score_pages' checks
    if (!q || !scores || !(scale > 0.0f) || !std::isfinite(scale)) return EKV_ERR_INVALID_ARG;
    if (policy != EKV_SEL_TOPK && policy != EKV_SEL_GAUSS && policy != EKV_SEL_GAUSS_MAX)
        return EKV_ERR_UNSUPPORTED;
    const bool gauss = policy != EKV_SEL_TOPK;
    if (gauss && !c->meta_mom) return EKV_ERR_INVALID_ARG;
    if ((uintptr_t)c->meta_bbox & 15u) return EKV_ERR_INVALID_ARG;
    if (gauss && ((uintptr_t)c->meta_mom & 15u)) return EKV_ERR_INVALID_ARG;
    return cuda_status(launch_refresh_score_pages(*c, new_start, new_count, max_new, q,
                                                  num_q_heads, scale, policy, scores,
                                                  static_cast<cudaStream_t>(stream), use_pdl()));
}

ekv_status ekv_select_pages(const ekv_cache *c, int32_t num_q_heads, int32_t policy,
                            int32_t topk, float alpha, float delta, const float *scores,
                            int32_t *sel_idx, int32_t *sel_count, int32_t max_sel,
                            float *tau_hat, void *stream)
{
    ekv_status s = check_cache(c, false);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    if (!scores || !sel_idx || !sel_count || max_sel < 1) return EKV_ERR_INVALID_ARG;
    if ((uintptr_t)scores & 15u) return EKV_ERR_INVALID_ARG;  // score rows are read as float4
    if (policy == EKV_SEL_TOPK) {
        if (topk < 1) return EKV_ERR_INVALID_ARG;
        const int need = topk < c->max_pages ? topk : c->max_pages;
        if (max_sel < need) return EKV_ERR_INVALID_ARG;
    } else if (policy == EKV_SEL_GAUSS || policy == EKV_SEL_GAUSS_MAX) {
        if (alpha != 1.5f && alpha != 2.0f) return EKV_ERR_UNSUPPORTED;
        if (!tau_hat || !std::isfinite(delta)) return EKV_ERR_INVALID_ARG;
    } else {
        return EKV_ERR_UNSUPPORTED;
    }
    return cuda_status(launch_select_pages(*c, num_q_heads, policy, topk, alpha, delta, scores,
                                           sel_idx, sel_count, max_sel, tau_hat,
                                           static_cast<cudaStream_t>(stream), use_pdl()));
}

ekv_status ekv_score_select_pages(const ekv_cache *c, const void *q, int32_t num_q_heads,
                                  float scale, int32_t topk, float *scores, int32_t *sel_idx,
                                  int32_t *sel_count, int32_t max_sel, void *stream)
{
    ekv_status s = check_cache(c, false);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    if (!q || !sel_idx || !sel_count || max_sel < 1 || topk < 1 || !(scale > 0.0f) ||
        !std::isfinite(scale))
        return EKV_ERR_INVALID_ARG;
    if (max_sel < (topk < c->max_pages ? topk : c->max_pages)) return EKV_ERR_INVALID_ARG;
    if ((uintptr_t)c->meta_bbox & 15u) return EKV_ERR_INVALID_ARG;
    if (scores && ((uintptr_t)scores & 15u)) return EKV_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (step_score_select_supported(*c))
        return cuda_status(launch_step_score_select(*c, q, num_q_heads, scale, topk, scores, sel_idx,
                                                    sel_count, max_sel, st, use_pdl()));
    // a geometry the cluster kernel does not hold: the two kernels, scores through global memory
    if (!scores) return EKV_ERR_INVALID_ARG;
    cudaError_t e = launch_score_pages(*c, q, num_q_heads, scale, EKV_SEL_TOPK, scores, st, use_pdl());
    if (e == cudaSuccess)
        e = launch_select_pages(*c, num_q_heads, EKV_SEL_TOPK, topk, 1.5f, 0.0f, scores, sel_idx,
                                sel_count, max_sel, nullptr, st, use_pdl());
    return cuda_status(e);
}

size_t ekv_decode_workspace_bytes(const ekv_cache *c, int32_t num_q_heads, int32_t max_sel)
{
    if (check_cache(c, false) != EKV_OK || check_heads(c, num_q_heads) != EKV_OK || max_sel < 1)
        return 0;
    return decode_workspace_bytes_all_modes(c->batch, num_q_heads, c->num_kv_heads, c->head_dim,
                                            c->page_size, c->dtype, max_sel);
}

ekv_status ekv_sparse_decode(const ekv_cache *c, const void *q, int32_t num_q_heads,
                             float scale, int32_t attn, const int32_t *sel_idx,
                             const int32_t *sel_count, int32_t max_sel, float *out, float *stat,
                             void *ws, size_t ws_bytes, void *stream)
{
    ekv_status s = check_cache(c, true);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    if (attn != EKV_SOFTMAX && attn != EKV_ENTMAX15 && attn != EKV_SPARSEMAX)
        return EKV_ERR_UNSUPPORTED;
    if (!q || !sel_idx || !sel_count || !out || !stat || max_sel < 1 || !(scale > 0.0f) ||
        !std::isfinite(scale))
        return EKV_ERR_INVALID_ARG;
    // K/V page spans and the query rows are moved with bulk copies: 16-byte aligned bases
    if (((uintptr_t)q | (uintptr_t)c->k_cache | (uintptr_t)c->v_cache) & 15u)
        return EKV_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ekv_decode_workspace_bytes(c, num_q_heads, max_sel))
        return EKV_ERR_WORKSPACE;
    if ((uintptr_t)ws & 15u) return EKV_ERR_INVALID_ARG;  // logits are read back as float4
    return cuda_status(launch_sparse_decode(*c, q, num_q_heads, scale, attn, sel_idx, sel_count,
                                            max_sel, out, stat, ws,
                                            static_cast<cudaStream_t>(stream), use_pdl()));
}

ekv_status ekv_select_decode(const ekv_cache *c, const void *q, int32_t num_q_heads, float scale,
                             int32_t attn, int32_t topk, const float *scores, int32_t *sel_idx,
                             int32_t *sel_count, int32_t max_sel, float *out, float *stat,
                             void *ws, size_t ws_bytes, void *stream)
{
    ekv_status s = check_cache(c, true);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    if (attn != EKV_SOFTMAX && attn != EKV_ENTMAX15 && attn != EKV_SPARSEMAX)
        return EKV_ERR_UNSUPPORTED;
    if (!q || !scores || !sel_idx || !sel_count || !out || !stat || max_sel < 1 || topk < 1 ||
        !(scale > 0.0f) || !std::isfinite(scale))
        return EKV_ERR_INVALID_ARG;
    if (max_sel < (topk < c->max_pages ? topk : c->max_pages)) return EKV_ERR_INVALID_ARG;
    if (((uintptr_t)scores | (uintptr_t)q | (uintptr_t)c->k_cache | (uintptr_t)c->v_cache) & 15u)
        return EKV_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ekv_decode_workspace_bytes(c, num_q_heads, max_sel))
        return EKV_ERR_WORKSPACE;
    if ((uintptr_t)ws & 15u) return EKV_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the selection kernel, then the decode launched behind it (programmatic dependent launch):
    // the decode's thread-block clusters are placed while the selection runs
    cudaError_t e = launch_select_pages(*c, num_q_heads, EKV_SEL_TOPK, topk, 1.5f, 0.0f, scores, sel_idx,
                            sel_count, max_sel, nullptr, st, use_pdl());
    if (e == cudaSuccess)
        e = launch_sparse_decode(*c, q, num_q_heads, scale, attn, sel_idx, sel_count, max_sel, out,
                                 stat, ws, st, use_pdl());
    return cuda_status(e);
}

size_t ekv_moment_bytes(const ekv_cache *c)
{
    if (check_cache(c, true) != EKV_OK) return 0;
    return (size_t)c->batch * c->num_kv_heads * EKV_MOMENT_FLOATS((size_t)c->head_dim) * sizeof(float);
}

ekv_status ekv_moment_update(const ekv_cache *c, float *moments, const int32_t *new_start,
                             const int32_t *new_count, int32_t max_new, void *stream)
{
    ekv_status s = check_cache(c, true);
    if (s != EKV_OK) return s;
    if (!moments || !new_start || !new_count || max_new < 0) return EKV_ERR_INVALID_ARG;
    if ((long long)max_new > (long long)c->max_pages * c->page_size) return EKV_ERR_INVALID_ARG;
    return cuda_status(launch_moment_update(*c, moments, new_start, new_count, max_new,
                                            static_cast<cudaStream_t>(stream)));
}

// The decode workspace, then (256-byte aligned) the sums over the selected tokens.
static size_t moment_ret_offset(size_t decode_bytes) { return (decode_bytes + 255) & ~(size_t)255; }

size_t ekv_moment_decode_workspace_bytes(const ekv_cache *c, int32_t num_q_heads, int32_t max_sel)
{
    const size_t base = ekv_decode_workspace_bytes(c, num_q_heads, max_sel);
    if (!base) return 0;
    return moment_ret_offset(base) + moment_retained_bytes(c->batch, c->num_kv_heads, c->head_dim,
                                                           num_q_heads / c->num_kv_heads);
}

ekv_status ekv_sparse_decode_moment(const ekv_cache *c, const float *moments, const void *q,
                                    int32_t num_q_heads, float scale, const int32_t *sel_idx,
                                    const int32_t *sel_count, int32_t max_sel, float *out,
                                    float *stat, void *ws, size_t ws_bytes, void *stream)
{
    ekv_status s = check_cache(c, true);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    if (!moments || !q || !sel_idx || !sel_count || !out || !stat || max_sel < 1 ||
        !(scale > 0.0f) || !std::isfinite(scale))
        return EKV_ERR_INVALID_ARG;
    if (((uintptr_t)q | (uintptr_t)c->k_cache | (uintptr_t)c->v_cache) & 15u)
        return EKV_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ekv_moment_decode_workspace_bytes(c, num_q_heads, max_sel))
        return EKV_ERR_WORKSPACE;
    if ((uintptr_t)ws & 15u) return EKV_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *ret = reinterpret_cast<float *>(
        static_cast<char *>(ws) + moment_ret_offset(ekv_decode_workspace_bytes(c, num_q_heads, max_sel)));
    cudaError_t e = launch_moment_pass(*c, moments, q, num_q_heads, scale, sel_idx, sel_count,
                                       max_sel, ret, out, stat, st, false);
    if (e == cudaSuccess)
        e = launch_sparse_decode(*c, q, num_q_heads, scale, EKV_SOFTMAX, sel_idx, sel_count,
                                 max_sel, out, stat, ws, st, use_pdl());
    if (e == cudaSuccess)
        e = launch_moment_pass(*c, moments, q, num_q_heads, scale, sel_idx, sel_count, max_sel,
                               ret, out, stat, st, true);
    return cuda_status(e);
}

size_t ekv_token_workspace_bytes(const ekv_cache *c, int32_t max_sel)
{
    if (check_cache(c, false) != EKV_OK || max_sel < 1) return 0;
    return (size_t)c->batch * c->num_kv_heads * max_sel * c->page_size * sizeof(float);
}

ekv_status ekv_select_tokens(const ekv_cache *c, const void *q, int32_t num_q_heads, float scale,
                             const int32_t *sel_idx, const int32_t *sel_count, int32_t max_sel,
                             int32_t T, int32_t *tok_page, int32_t *tok_pos, int32_t *tok_count,
                             void *ws, size_t ws_bytes, void *stream)
{
    ekv_status s = check_cache(c, false);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    if (!q || !sel_idx || !sel_count || !tok_page || !tok_pos || !tok_count || max_sel < 1 ||
        T < 1 || !(scale > 0.0f) || !std::isfinite(scale))
        return EKV_ERR_INVALID_ARG;
    if (T > EKV_MAX_TOKENS) return EKV_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < ekv_token_workspace_bytes(c, max_sel)) return EKV_ERR_WORKSPACE;
    if ((uintptr_t)ws & 15u) return EKV_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *tscores = static_cast<float *>(ws);
    cudaError_t e = launch_token_scores(*c, q, num_q_heads, scale, sel_idx, sel_count, max_sel,
                                        tscores, st);
    if (e == cudaSuccess)
        e = launch_select_tokens(*c, tscores, sel_idx, sel_count, max_sel, T, tok_page, tok_pos,
                                 tok_count, st);
    return cuda_status(e);
}

ekv_status ekv_sparse_decode_tokens(const ekv_cache *c, const void *q, int32_t num_q_heads,
                                    float scale, int32_t attn, const int32_t *tok_page,
                                    const int32_t *tok_pos, const int32_t *tok_count, int32_t T,
                                    float *out, float *stat, void *stream)
{
    ekv_status s = check_cache(c, true);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    if (attn != EKV_SOFTMAX && attn != EKV_ENTMAX15 && attn != EKV_SPARSEMAX)
        return EKV_ERR_UNSUPPORTED;
    if (!q || !tok_page || !tok_pos || !tok_count || !out || !stat || T < 1 || !(scale > 0.0f) ||
        !std::isfinite(scale))
        return EKV_ERR_INVALID_ARG;
    if (T > EKV_MAX_TOKENS) return EKV_ERR_UNSUPPORTED;
    return cuda_status(launch_token_attend(*c, q, num_q_heads, scale, attn, tok_page, tok_pos,
                                           tok_count, T, out, stat,
                                           static_cast<cudaStream_t>(stream)));
}

ekv_status ekv_selection_quality(const ekv_cache *c, const void *q, int32_t num_q_heads,
                                 float scale, int32_t attn, const float *stat_full,
                                 const int32_t *sel_idx, const int32_t *sel_count,
                                 int32_t max_sel, double *dropped, int32_t *support, void *stream)
{
    ekv_status s = check_cache(c, false);
    if (s != EKV_OK) return s;
    if ((s = check_heads(c, num_q_heads)) != EKV_OK) return s;
    if (attn != EKV_SOFTMAX && attn != EKV_ENTMAX15 && attn != EKV_SPARSEMAX)
        return EKV_ERR_UNSUPPORTED;
    if (!q || !stat_full || !sel_idx || !sel_count || !dropped || !support || max_sel < 1 ||
        !(scale > 0.0f) || !std::isfinite(scale))
        return EKV_ERR_INVALID_ARG;
    return cuda_status(launch_selection_quality(*c, q, num_q_heads, scale, attn, stat_full,
                                                sel_idx, sel_count, max_sel, dropped, support,
                                                static_cast<cudaStream_t>(stream)));
}

ekv_status ekv_device_status(const ekv_cache *c, uint32_t *bits, void *stream)
{
    if (!c || !c->dev_status) return EKV_ERR_INVALID_ARG;
    uint32_t h = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&h, c->dev_status, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return EKV_ERR_CUDA;
    if (bits) *bits = h;
    return h ? EKV_ERR_DEVICE : EKV_OK;
}

ekv_status ekv_clear_device_status(const ekv_cache *c, void *stream)
{
    if (!c || !c->dev_status) return EKV_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(c->dev_status, 0, sizeof(uint32_t),
                                       static_cast<cudaStream_t>(stream)));
}

ekv_status ekv_wait_selftest(const ekv_cache *c, uint64_t limit_ns, void *stream)
{
    if (!c || !c->dev_status || limit_ns > 2000000000ull) return EKV_ERR_INVALID_ARG;
    return cuda_status(launch_wait_selftest(c->dev_status, limit_ns, static_cast<cudaStream_t>(stream)));
}

const char *ekv_status_str(ekv_status s)
{
    switch (s) {
    case EKV_OK: return "EKV_OK";
    case EKV_ERR_INVALID_ARG: return "EKV_ERR_INVALID_ARG";
    case EKV_ERR_UNSUPPORTED: return "EKV_ERR_UNSUPPORTED";
    case EKV_ERR_WORKSPACE: return "EKV_ERR_WORKSPACE";
    case EKV_ERR_CUDA: return "EKV_ERR_CUDA";
    case EKV_ERR_DEVICE: return "EKV_ERR_DEVICE";
    }
    return "EKV_UNKNOWN_STATUS";
}

}  // extern "C"
