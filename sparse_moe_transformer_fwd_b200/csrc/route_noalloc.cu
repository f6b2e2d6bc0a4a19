// moe_route_noalloc: the router (router_scores + router_topk kernels of
// router.cu) with its [T, E] score scratch in a fixed device array of this
// library instead of a caller workspace, for callers that may not allocate
// device memory.  See include/moe_fwd.h for the contract (size limit, first
// call per device, races between overlapping calls).
#include "common.cuh"
#include "kernels.h"

#include <cstdio>
#include <mutex>

namespace moe {
namespace {

// Score scratch shared by every call; each call overwrites the T*E entries it
// reads, so nothing needs clearing between calls.
static __device__ __align__(256) float g_noalloc_scores[MOE_ROUTE_NOALLOC_MAX_SCORES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float *g_addr[kMaxDevices] = {};
unsigned long long g_ctx_id[kMaxDevices] = {};  // context the address was looked up in

thread_local char g_msg[256];

// Device address of the scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, once per device and context: a device whose primary
// context was destroyed (cudaDeviceReset) and created again loads the
// library's module anew, possibly at another address, so a new context id
// repeats the lookup (as does a driver that cannot report ids: id 0).
cudaError_t scratch_address(float **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev] || id == 0 || id != g_ctx_id[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scores);
        if (e != cudaSuccess) return e;
        g_addr[dev] = static_cast<float *>(p);
        // the lookup made the device's primary context current if none was
        g_ctx_id[dev] = current_context_id();
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" int moe_route_noalloc(const moe_shape *s, const uint16_t *x, const uint16_t *w_router,
                                 const float *bias, int32_t *topk_idx, float *topk_w,
                                 void *stream) {
    using namespace moe;
    const CallRange nvtx_range("moe_route_noalloc");
    if (!s) return record_error(MOE_ERR_INVALID_ARG, "shape is NULL");
    const int rc = validate_shape(s);
    if (rc != MOE_OK) return rc;
    const long long n = static_cast<long long>(s->T) * s->n_experts;
    if (n > MOE_ROUTE_NOALLOC_MAX_SCORES) {
        snprintf(g_msg, sizeof g_msg,
                 "moe_route_noalloc: T * n_experts = %lld exceeds the fixed scratch of %d scores",
                 n, MOE_ROUTE_NOALLOC_MAX_SCORES);
        return record_error(MOE_ERR_INVALID_ARG, g_msg);
    }
    if (s->T == 0) {
        record_launches(0);
        return MOE_OK;
    }
    const void *ptrs[] = {x, w_router, bias, topk_idx, topk_w};
    const char *names[] = {"x", "w_router", "bias", "topk_idx", "topk_w"};
    for (int i = 0; i < 5; ++i) {
        if (!ptrs[i] || (reinterpret_cast<uintptr_t>(ptrs[i]) & 15)) {
            snprintf(g_msg, sizeof g_msg, "%s is NULL or not 16-byte aligned", names[i]);
            return record_error(MOE_ERR_INVALID_ARG, g_msg);
        }
    }
    // the same device check (and error code) as moe_route
    const int dc = validate_device();
    if (dc != MOE_OK) return dc;
    float *scores = nullptr;
    cudaError_t e = scratch_address(&scores);
    if (e != cudaSuccess) {
        snprintf(g_msg, sizeof g_msg, "moe_route_noalloc: scratch address: %s",
                 cudaGetErrorString(e));
        return record_error(MOE_ERR_CUDA, g_msg);
    }
    int launches = 0;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    e = launch_router(x, w_router, bias, s->T, s->d_model, s->n_experts, s->top_k,
                      s->routed_scale, scores, topk_idx, topk_w, st, &launches);
    if (e != cudaSuccess) {
        snprintf(g_msg, sizeof g_msg, "moe_route_noalloc: %s", cudaGetErrorString(e));
        return record_error(MOE_ERR_CUDA, g_msg);
    }
    mark_launch(st, launches);
    record_launches(launches);
    return MOE_OK;
}
