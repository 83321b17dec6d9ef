// topk_noalloc.cu -- v4a_topk for callers that cannot allocate device memory.
//
// v4a_topk needs a caller-provided workspace (it holds the fp32 indexer
// scores between the scoring and the select kernels).  Some callers have no
// way to obtain one: a plug-in that runs inside a host framework which owns
// every device allocation and hands out none, or a latency-critical serving
// loop where an allocation (or a trip through a caching allocator) is not
// allowed.  v4a_topk_noalloc gives them the same operation with the scratch
// taken from a fixed array compiled into this library instead.
//
// The array lives in device global memory for as long as the library is
// loaded on a device; its host-side name is only a stand-in, so its device
// address is looked up once per device with cudaGetSymbolAddress and cached
// (for the device's current context: a cudaDeviceReset makes it stale).
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = 64u << 20;  // 64 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_topk_scratch[kScratchBytes];

std::mutex g_lock;
void* g_scratch_addr[kMaxDevices] = {};

// The device address of g_topk_scratch on the current device (set up on the
// first call made with that device current).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> g(g_lock);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_topk_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" v4a_status v4a_topk_noalloc(const void* q_i, const float* w, const void* k_i, const float* k_scale,
                                       int32_t* idx_out, float* score_out, int heads_i, int d_i, v4a_dtype q_dtype,
                                       v4a_dtype k_dtype, const v4a_shape* shape, void* stream) {
    if (!shape) return v4a::report(V4A_ERR_INVALID_ARG, "shape is NULL");
    if (shape->batch < 0 || shape->n_q < 1 || shape->ctx_len < 0 || shape->m < 1 || shape->k < 1)
        // not a shape v4a_topk takes, so no scratch size applies: v4a_topk's own checks say why (it
        // rejects the shape before looking at the scratch, and launches nothing)
        return v4a_topk(q_i, w, k_i, k_scale, idx_out, score_out, heads_i, d_i, q_dtype, k_dtype, nullptr, 0, shape,
                        stream);
    const size_t need = v4a_workspace_size("topk", shape, heads_i, d_i);
    if (need > kScratchBytes)
        return v4a::report(V4A_ERR_INVALID_ARG,
                           "v4a_topk_noalloc: this shape needs %zu bytes of scratch (v4a_workspace_size \"topk\") "
                           "but the built-in array holds %zu; use v4a_topk with a workspace",
                           need, kScratchBytes);
    void* scratch = nullptr;
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess)
        return v4a::report(V4A_ERR_CUDA, "v4a_topk_noalloc: scratch set-up: %s", cudaGetErrorString(e));
    // same checks and kernels as v4a_topk; only the scratch differs
    return v4a_topk(q_i, w, k_i, k_scale, idx_out, score_out, heads_i, d_i, q_dtype, k_dtype, scratch, kScratchBytes,
                    shape, stream);
}
