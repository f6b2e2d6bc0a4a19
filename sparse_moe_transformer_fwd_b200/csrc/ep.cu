// Expert parallelism: the dispatch of one source rank's permuted rows into
// the owners' receive buffers ("DeepSeek v3 and R1 Model Architecture",
// "Local Balanced Routing to Experts": experts are spread over devices and
// tokens travel to the devices that hold their experts).
//
// A source rank's routed rows are in global expert order, so the rows for
// owner o (experts o*P .. o*P + P - 1) are one contiguous block; each block
// is copied with 16-byte stores (and its fp32 block scales with 4-byte ones)
// to the given destination pointer, which may be another GPU's memory (a
// peer mapping) or, for several ranks emulated on one GPU, a buffer of this
// one.  No TMA, no multicast: plain loads of this GPU's memory and plain
// stores.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// One CTA per row (grid-stride): the row's block by a scan of the block
// prefix (at most kMaxEpRanks blocks), then its bytes and scales.
__global__ void __launch_bounds__(128)
ep_dispatch_kernel(const uint8_t *__restrict__ a, const float *__restrict__ a_s,
                   const EpDispatchArgs g) {
    pdl_wait_and_trigger();
    const int R = g.prefix[g.n_blocks];
    const int nvec = g.row_bytes / 16;
    for (int r = blockIdx.x; r < R; r += gridDim.x) {
        int b = 0;
        while (b + 1 < g.n_blocks && g.prefix[b + 1] <= r) ++b;
        const int off = r - g.prefix[b];
        const size_t src = static_cast<size_t>(g.src_row[b]) + off;
        const size_t dst = static_cast<size_t>(g.dst_row[b]) + off;
        const uint4 *s4 = reinterpret_cast<const uint4 *>(a + src * g.row_bytes);
        uint4 *d4 = reinterpret_cast<uint4 *>(g.dst_a[g.dst[b]] + dst * g.row_bytes);
        for (int i = threadIdx.x; i < nvec; i += blockDim.x) d4[i] = __ldg(s4 + i);
        if (a_s) {
            const float *ss = a_s + src * g.n_scales;
            float *ds = g.dst_s[g.dst[b]] + dst * g.n_scales;
            for (int i = threadIdx.x; i < g.n_scales; i += blockDim.x) ds[i] = __ldg(ss + i);
        }
    }
}

}  // namespace

cudaError_t launch_ep_dispatch(const void *a, const float *a_scales, const EpDispatchArgs &g,
                               cudaStream_t st, int *launches) {
    const int R = g.prefix[g.n_blocks];
    if (R <= 0) return cudaSuccess;
    const int grid = R < 8 * num_sms() ? R : 8 * num_sms();
    mark_launch(st, *launches, "ep_dispatch");
    LAUNCH_OR_RETURN(launch_pdl(ep_dispatch_kernel, dim3(grid), dim3(128), 0, st,
                                static_cast<const uint8_t *>(a), a_scales, g));
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
