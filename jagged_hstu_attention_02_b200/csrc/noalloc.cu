// noalloc.cu -- a forward entry point for callers that cannot allocate device memory.
//
// hstu_attn_fwd needs a caller-provided workspace (a status word plus an fp32 buffer for
// the per-token attention output before the LayerNorm).  Some callers have no way to
// provide one: a plugin hosted by a framework that owns all device memory and offers no
// allocation hook, or a latency-critical serving loop in which cudaMalloc (which can
// synchronise the whole device) is not allowed.  For them, hstu_attn_fwd_noalloc runs the
// same forward with its scratch taken from a fixed array in device memory that the library
// itself declares at file scope.  Every GPU that loads this library keeps that array for
// the lifetime of the process.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace hstu {
namespace {

// Fixed scratch: 32 MiB per device, enough for the forward of about 16k tokens at
// H * d_v = 512 (the need is 256 bytes + 4 * total_tokens * H * d_v bytes).
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices];                 // device address of the array, per device
unsigned long long g_noalloc_ctx[kMaxDevices];    // id of the context it was looked up in

// Unique id of the calling thread's current context (0 when it cannot be told).  A device
// reset destroys the context and, with it, the array's address; a new context gets a new
// id, so the address is looked up again.
unsigned long long current_context_id()
{
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    if (!get_current || !get_id) {
        void *a = nullptr, *b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
            qa != cudaDriverEntryPointSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
            qb != cudaDriverEntryPointSuccess)
            return 0;
        get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(a);
        get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(b);
    }
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array on the current device.  The name of a __device__
// array is only a host-side handle, so the address comes from cudaGetSymbolAddress, once
// per device (and again after that device's context was reset), with that device current.
hstu_status_t noalloc_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HSTU_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return HSTU_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
            return HSTU_ERR_CUDA;
        g_noalloc_ptr[dev] = ptr;
        g_noalloc_ctx[dev] = current_context_id();   // the lookup made the context current
    }
    *out = g_noalloc_ptr[dev];
    return HSTU_OK;
}

}  // namespace
}  // namespace hstu

extern "C" hstu_status_t hstu_attn_fwd_noalloc(const hstu_attn_params_t *params, const void *q,
                                               const void *k, const void *v, const void *u,
                                               const int64_t *seq_offsets,
                                               const int32_t *num_contextuals,
                                               const int32_t *num_targets,
                                               const int64_t *timestamps, const float *rel_bias,
                                               const float *time_bias, void *out, void *stream)
{
    size_t need = 0;
    hstu_status_t st = hstu_attn_fwd_workspace_size(params, &need);
    if (st != HSTU_OK) return st;
    if (need > hstu::kNoAllocScratchBytes) return HSTU_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = nullptr;
    st = hstu::noalloc_scratch(&scratch);
    if (st != HSTU_OK) return st;
    // Inference forward (no saved activations); the status word at the head of the scratch
    // is cleared by hstu_attn_fwd before its kernels run.
    return hstu_attn_fwd(params, q, k, v, u, seq_offsets, num_contextuals, num_targets, timestamps,
                         rel_bias, time_bias, out, nullptr, nullptr, nullptr, scratch,
                         hstu::kNoAllocScratchBytes, stream);
}
