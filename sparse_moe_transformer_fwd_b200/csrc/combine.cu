// Weighted un-permute and shared-expert add ("DeepSeek v3 and R1 Model
// Architecture", "Structural change": one always-activated shared expert):
//   out[t] = bf16( sum_j g[t,j] * Y[row_of[t,j]]  (rank order, binary32 fma)
//                  + Y[T*k + t]                   (shared, weight 1)
//                  [+ h[t]] )                     (residual of the pre-norm block)
// CTA (t, y) covers 16-byte vectors y*128 .. y*128+127 of token t's row, one
// per thread; the k + 1 (+ 1) source loads of a vector are issued together
// (groups of 8 routed rows) before the additions, which keep rank order.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int CB_THREADS = 128;

__device__ __forceinline__ void add8(float (&acc)[8], const uint4 raw) {
    const uint32_t r[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], bf16_lo(r[i]));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], bf16_hi(r[i]));
    }
}

__global__ void __launch_bounds__(CB_THREADS)
combine_kernel(const uint16_t *__restrict__ y, const int32_t *__restrict__ row_of,
               const float *__restrict__ gates, int T, int d, int k, int n_shared,
               uint16_t *__restrict__ out, const uint16_t *__restrict__ residual) {
    __shared__ int rows_sh[32];
    __shared__ float g_sh[32];
    const int t = blockIdx.x;
    const int v = blockIdx.y * CB_THREADS + threadIdx.x;
    pdl_wait_and_trigger();
    if (threadIdx.x < k) {
        rows_sh[threadIdx.x] = row_of[static_cast<size_t>(t) * k + threadIdx.x];
        g_sh[threadIdx.x] = gates[static_cast<size_t>(t) * k + threadIdx.x];
    }
    __syncthreads();
    if (v >= d / 8) return;
    uint4 raw_s = make_uint4(0, 0, 0, 0), raw_h = make_uint4(0, 0, 0, 0);
    if (n_shared)
        raw_s = reinterpret_cast<const uint4 *>(y + (static_cast<size_t>(T) * k + t) * d)[v];
    if (residual) raw_h = reinterpret_cast<const uint4 *>(residual + static_cast<size_t>(t) * d)[v];
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j0 = 0; j0 < k; j0 += 8) {
        uint4 raw[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
            if (j0 + jj < k)
                raw[jj] = reinterpret_cast<const uint4 *>(
                    y + static_cast<size_t>(rows_sh[j0 + jj]) * d)[v];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            if (j0 + jj >= k) break;
            const uint32_t r[4] = {raw[jj].x, raw[jj].y, raw[jj].z, raw[jj].w};
            const float g = g_sh[j0 + jj];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = __fmaf_rn(g, bf16_lo(r[i]), acc[2 * i]);
                acc[2 * i + 1] = __fmaf_rn(g, bf16_hi(r[i]), acc[2 * i + 1]);
            }
        }
    }
    if (n_shared) add8(acc, raw_s);
    if (residual) add8(acc, raw_h);  // pre-norm block: out = h + MoE(x), one final rounding
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    reinterpret_cast<uint4 *>(out + static_cast<size_t>(t) * d)[v] = o;
}

}  // namespace

cudaError_t launch_combine(const uint16_t *y, const int32_t *row_of, const float *gates, int T,
                           int d, int k, int n_shared, uint16_t *out, cudaStream_t st,
                           int *launches, const uint16_t *residual) {
    mark_launch(st, *launches, "combine");
    const dim3 grid(T, (d / 8 + CB_THREADS - 1) / CB_THREADS);
    LAUNCH_OR_RETURN(launch_pdl(combine_kernel, grid, dim3(CB_THREADS), 0, st, y, row_of, gates, T, d, k, n_shared,
                                out, residual));
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
