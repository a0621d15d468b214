// decode_noalloc.cu -- ekv_sparse_decode_noalloc: the sparse decode of ekv_sparse_decode with
// its scratch taken from a fixed array inside the library instead of a caller buffer.
//
// For callers that cannot allocate device memory: code whose allocator has already reserved
// all of HBM for the KV cache and its own pools, code that must not risk a synchronising
// cudaMalloc/cudaFree on a latency-critical path, and plug-ins that are handed only their
// inputs and outputs. The scratch is one file-scope __device__ array of
// EKV_NOALLOC_WS_BYTES bytes, present on every GPU that loads the library until the process
// exits. Its device address is looked up once per device (cudaGetSymbolAddress, with that
// device current) on the first call made on that device.
#include <mutex>

#include "ekv_device.cuh"

namespace ekv {
cudaError_t launch_sparse_decode(const ekv_cache &c, const void *q, int H_q, float scale,
                                 int attn, const int32_t *sel_idx, const int32_t *sel_count,
                                 int max_sel, float *out, float *stat, void *ws, cudaStream_t st,
                                 bool pdl);
}

// The shared scratch. Host code must not use this name as an address: on the host it is a
// stand-in object, not device memory. Only the address returned by cudaGetSymbolAddress may
// be handed to kernels.
static __device__ __align__(256) unsigned char g_noalloc_ws[EKV_NOALLOC_WS_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_ws_addr[kMaxDevices];  // device address of g_noalloc_ws, per device (null: not yet)

// The scratch's device address on the current device, looked up on first use.
cudaError_t noalloc_workspace(void **addr)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ws_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_ws);
        if (e != cudaSuccess) return e;
        g_ws_addr[dev] = p;
    }
    *addr = g_ws_addr[dev];
    return cudaSuccess;
}
}  // namespace

extern "C" ekv_status ekv_sparse_decode_noalloc(const ekv_cache *c, const void *q,
                                                int32_t num_q_heads, float scale, int32_t attn,
                                                const int32_t *sel_idx, const int32_t *sel_count,
                                                int32_t max_sel, float *out, float *stat,
                                                void *stream)
{
    const size_t need = ekv_decode_workspace_bytes(c, num_q_heads, max_sel);
    if (need == 0) {
        // invalid geometry: let the allocating entry point's checks name the problem
        return ekv_sparse_decode(c, q, num_q_heads, scale, attn, sel_idx, sel_count, max_sel, out,
                                 stat, nullptr, 0, stream);
    }
    if (need > (size_t)EKV_NOALLOC_WS_BYTES) return EKV_ERR_WORKSPACE;
    if (attn != EKV_SOFTMAX && attn != EKV_ENTMAX15 && attn != EKV_SPARSEMAX)
        return EKV_ERR_UNSUPPORTED;
    if (!q || !sel_idx || !sel_count || !out || !stat || !c->v_cache || !(scale > 0.0f) ||
        !(scale < INFINITY) || (((uintptr_t)q | (uintptr_t)c->k_cache | (uintptr_t)c->v_cache) & 15u))
        return EKV_ERR_INVALID_ARG;
    void *ws = nullptr;
    if (noalloc_workspace(&ws) != cudaSuccess) return EKV_ERR_CUDA;
    // Nothing in the scratch has to start at zero: every word a call reads was written
    // earlier in the same call.
    return ekv::launch_sparse_decode(*c, q, num_q_heads, scale, attn, sel_idx, sel_count, max_sel,
                                     out, stat, ws, static_cast<cudaStream_t>(stream),
                                     ekv::use_pdl()) ==
                   cudaSuccess
               ? EKV_OK
               : EKV_ERR_CUDA;
}
