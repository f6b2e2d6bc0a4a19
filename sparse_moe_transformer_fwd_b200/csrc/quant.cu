// Blockwise e4m3 quantisation ("DeepSeek-R1", aguasto.com, "Quantization":
// the checkpoint is blockwise FP8).  Per tile: amax = max |v| (exact on the
// bf16 inputs), scale = amax / 448 and inv = 448 / amax (correctly rounded
// binary32 divisions), code = e4m3 round-to-nearest-even, saturating, of the
// binary32 product v * inv (hardware cvt.rn.satfinite.e4m3x2.f32).  An
// all-zero tile gets scale 1 and +0 codes.  UE8M0 variant (flag ue): the
// scale is the least power of two 2^k (k >= -127) with amax / 2^k <= 448 and
// inv = 2^-k, so v * inv is exact and no code saturates.
//
// Activations use 1x128 tiles: 16 threads own one tile (8 elements each,
// one 16-byte load), amax by shuffles inside the 16-lane group.  Weights use
// 128x128 blocks: one CTA per block, 64 elements per thread in registers,
// amax through shared memory.  The forward pass fuses activation
// quantisation with the permutation: each token row is quantised once and
// its codes and scales are written to its k routed rows and its shared row.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

struct Quant8 {
    float v[8];
};

__device__ __forceinline__ Quant8 load8_bf16(const uint16_t *p) {
    const uint4 raw = *reinterpret_cast<const uint4 *>(p);
    const uint32_t r[4] = {raw.x, raw.y, raw.z, raw.w};
    Quant8 q;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        q.v[2 * i] = bf16_lo(r[i]);
        q.v[2 * i + 1] = bf16_hi(r[i]);
    }
    return q;
}

__device__ __forceinline__ float amax8(const Quant8 &q) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(q.v[i]));
    return m;
}

// codes of 8 values for a tile with the given amax; returns the scale
// (ue: the power-of-two UE8M0 scale instead of amax / 448)
__device__ __forceinline__ uint2 encode8(const Quant8 &q, float amax, float *scale, bool ue) {
    if (amax == 0.0f) {
        *scale = 1.0f;
        return make_uint2(0, 0);
    }
    float inv;
    if (ue) {
        *scale = ue8m0_scale(amax, &inv);
    } else {
        *scale = __fdiv_rn(amax, 448.0f);
        inv = __fdiv_rn(448.0f, amax);
    }
    uint16_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] = e4m3x2(__fmul_rn(q.v[2 * i], inv), __fmul_rn(q.v[2 * i + 1], inv));
    return make_uint2(static_cast<uint32_t>(c[0]) | (static_cast<uint32_t>(c[1]) << 16),
                      static_cast<uint32_t>(c[2]) | (static_cast<uint32_t>(c[3]) << 16));
}

__device__ __forceinline__ float group16_max(float m) {
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    return m;
}

// 1 x 128 tiles over a [rows, cols] matrix
__global__ void __launch_bounds__(256)
quant_1x128_kernel(const uint16_t *__restrict__ in, int rows, int cols, int ld,
                   uint8_t *__restrict__ q, float *__restrict__ scales, int ue) {
    pdl_wait_and_trigger();
    const int vpr = cols / 8;  // 16-byte vectors per row
    const long long total = static_cast<long long>(rows) * vpr;
    const long long nthreads = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long base = static_cast<long long>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
         base < total; base += nthreads) {
        const long long v = base + (threadIdx.x & 31);
        const bool ok = v < total;
        const int r = ok ? static_cast<int>(v / vpr) : 0;
        const int vc = ok ? static_cast<int>(v % vpr) : 0;
        Quant8 x;
        if (ok) x = load8_bf16(in + static_cast<size_t>(r) * ld + vc * 8);
        else
#pragma unroll
            for (int i = 0; i < 8; ++i) x.v[i] = 0.0f;
        const float amax = group16_max(amax8(x));
        float sc;
        const uint2 codes = encode8(x, amax, &sc, ue);
        if (ok) {
            *reinterpret_cast<uint2 *>(q + static_cast<size_t>(r) * cols + vc * 8) = codes;
            if ((vc & 15) == 0) scales[static_cast<size_t>(r) * (cols / 128) + vc / 16] = sc;
        }
    }
}

// 128 x 128 blocks; one CTA (256 threads) per block, grid-stride over blocks.
// tiled: block (rb, kb) is written as one contiguous 16 KB tile (128 rows of
// 128 codes) at tile index rb * (cols/128) + kb.
__global__ void __launch_bounds__(256)
quant_128x128_kernel(const uint16_t *__restrict__ in, int rows, int cols, int ld, int tiled,
                     uint8_t *__restrict__ q, float *__restrict__ scales, int ue) {
    __shared__ float red[8];
    pdl_wait_and_trigger();
    const int nkb = cols / 128, nrb = (rows + 127) / 128;
    const long long nblocks = static_cast<long long>(nkb) * nrb;
    const int tr = threadIdx.x / 16, tc = (threadIdx.x % 16) * 8;
    for (long long b = blockIdx.x; b < nblocks; b += gridDim.x) {
        const int rb = static_cast<int>(b / nkb), kb = static_cast<int>(b % nkb);
        Quant8 x[8];
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = rb * 128 + tr + 16 * i;
            if (r < rows) x[i] = load8_bf16(in + static_cast<size_t>(r) * ld + kb * 128 + tc);
            else
#pragma unroll
                for (int j = 0; j < 8; ++j) x[i].v[j] = 0.0f;
            m = fmaxf(m, amax8(x[i]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
        __syncthreads();
        float amax = red[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
        __syncthreads();
        float sc = 1.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = rb * 128 + tr + 16 * i;
            const uint2 codes = encode8(x[i], amax, &sc, ue);
            const size_t at = tiled ? (static_cast<size_t>(b) << 14) + (tr + 16 * i) * 128 + tc
                                    : static_cast<size_t>(r) * cols + kb * 128 + tc;
            if (r < rows) *reinterpret_cast<uint2 *>(q + at) = codes;
        }
        if (threadIdx.x == 0) scales[static_cast<size_t>(rb) * nkb + kb] = sc;
    }
}

// Pre-norm statistics ("DeepSeek-R1" card, "Facts": pre-norm RMSNorm before
// the MLP): one warp per token; lane l sums h_i^2 over i = l (mod 32) with
// fused multiply-adds in ascending i, five xor-butterfly rounds add the 32
// partial sums (every lane ends with the same value), then
// rstd = 1 / sqrt(S / d + eps), each step a correctly rounded binary32 op.
__global__ void __launch_bounds__(256)
rstd_kernel(const uint16_t *__restrict__ h, int T, int d, float eps, float *__restrict__ rstd) {
    pdl_wait_and_trigger();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const uint16_t *row = h + static_cast<size_t>(t) * d;
    float acc = 0.0f;
    for (int i = lane; i < d; i += 32) {
        const float v = __uint_as_float(static_cast<uint32_t>(row[i]) << 16);
        acc = __fmaf_rn(v, v, acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
    if (lane == 0) {
        const float mean = __fdiv_rn(acc, static_cast<float>(d));
        rstd[t] = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
    }
}

// x values of 8 consecutive columns c0.. of token t: bf16 inputs, or the
// pre-norm of the residual stream h when rstd is set.
__device__ __forceinline__ Quant8 load8_x(const uint16_t *row, int c0, float rstd,
                                          const uint16_t *gamma) {
    Quant8 v = load8_bf16(row + c0);
    if (gamma) {
        const Quant8 g = load8_bf16(gamma + c0);
#pragma unroll
        for (int i = 0; i < 8; ++i) v.v[i] = prenorm_elem(v.v[i], rstd, g.v[i]);
    }
    return v;
}

// Forward pass: quantise token t's row once, write it to its k + n_shared rows.
__global__ void __launch_bounds__(256)
quant_scatter_kernel(const uint16_t *__restrict__ x, int T, int d, int k, int n_shared,
                     const int32_t *__restrict__ row_of, uint8_t *__restrict__ a,
                     float *__restrict__ a_scales, PreNorm pn, int ue) {
    __shared__ int rows_sh[33];
    const int t = blockIdx.x;
    const int ndst = k + n_shared;
    pdl_wait_and_trigger();
    if (threadIdx.x < k) rows_sh[threadIdx.x] = row_of[static_cast<size_t>(t) * k + threadIdx.x];
    if (threadIdx.x == 0 && n_shared) rows_sh[k] = T * k + t;
    __syncthreads();
    const int ntiles = d / 128, nkb = d / 128;
    const int g = threadIdx.x / 16, l16 = threadIdx.x % 16;
    const float rs = pn.rstd ? pn.rstd[t] : 1.0f;
    // CTA (t, y) quantises tiles 16y .. 16y+15 of the row (16 threads per tile)
    const int tile = blockIdx.y * 16 + g;
    const bool ok = tile < ntiles;
    Quant8 v;
    if (ok) v = load8_x(x + static_cast<size_t>(t) * d, tile * 128 + l16 * 8, rs, pn.gamma);
    else
#pragma unroll
        for (int i = 0; i < 8; ++i) v.v[i] = 0.0f;
    const float amax = group16_max(amax8(v));
    float sc;
    const uint2 codes = encode8(v, amax, &sc, ue);
    if (!ok) return;
    for (int j = 0; j < ndst; ++j) {
        const size_t row = static_cast<size_t>(rows_sh[j]);
        *reinterpret_cast<uint2 *>(a + row * d + tile * 128 + l16 * 8) = codes;
        if (l16 == 0) a_scales[row * nkb + tile] = sc;
    }
}

__global__ void __launch_bounds__(256)
scatter_bf16_kernel(const uint16_t *__restrict__ x, int T, int d, int k, int n_shared,
                    const int32_t *__restrict__ row_of, uint16_t *__restrict__ a, PreNorm pn) {
    __shared__ int rows_sh[33];
    const int t = blockIdx.x;
    const int ndst = k + n_shared;
    pdl_wait_and_trigger();
    if (threadIdx.x < k) rows_sh[threadIdx.x] = row_of[static_cast<size_t>(t) * k + threadIdx.x];
    if (threadIdx.x == 0 && n_shared) rows_sh[k] = T * k + t;
    __syncthreads();
    const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t) * d);
    const float rs = pn.rstd ? pn.rstd[t] : 1.0f;
    // CTA (t, y) copies 16-byte vectors 256y .. 256y+255 of the row
    for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < min(d / 8, (blockIdx.y + 1) * blockDim.x);
         v += blockDim.x) {
        uint4 val = make_uint4(0, 0, 0, 0);
        if (!pn.gamma) val = src[v];
        else {
            const Quant8 xv = load8_x(x + static_cast<size_t>(t) * d, v * 8, rs, pn.gamma);
            val.x = pack_bf16x2(xv.v[0], xv.v[1]);
            val.y = pack_bf16x2(xv.v[2], xv.v[3]);
            val.z = pack_bf16x2(xv.v[4], xv.v[5]);
            val.w = pack_bf16x2(xv.v[6], xv.v[7]);
        }
        for (int j = 0; j < ndst; ++j)
            reinterpret_cast<uint4 *>(a + static_cast<size_t>(rows_sh[j]) * d)[v] = val;
    }
}

// Row-major rows x row_bytes -> 128 x 128-byte tiles; one 16-byte vector per
// thread and step, grid-stride.
__global__ void __launch_bounds__(256)
pack_tiles_kernel(const uint8_t *__restrict__ src, int rows, int row_bytes,
                  uint8_t *__restrict__ dst) {
    pdl_wait_and_trigger();
    const int tpr = row_bytes / 128;                       // tiles per row band
    const long long total = static_cast<long long>(rows) * (row_bytes / 16);
    for (long long v = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; v < total;
         v += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int r = static_cast<int>(v / (row_bytes / 16));
        const int cb = static_cast<int>(v % (row_bytes / 16)) * 16;   // byte column
        const size_t tile = static_cast<size_t>(r / 128) * tpr + cb / 128;
        const uint4 val = *reinterpret_cast<const uint4 *>(src + static_cast<size_t>(r) * row_bytes + cb);
        *reinterpret_cast<uint4 *>(dst + (tile << 14) + (r % 128) * 128 + (cb % 128)) = val;
    }
}

}  // namespace

cudaError_t launch_pack_tiles(const void *src, int rows, int row_bytes, void *dst, cudaStream_t st,
                              int *launches) {
    const long long total = static_cast<long long>(rows) * (row_bytes / 16);
    const long long want = (total + 255) / 256;
    const int grid = static_cast<int>(want < num_sms() * 16LL ? want : num_sms() * 16LL);
    mark_launch(st, *launches, "pack_tiles");
    LAUNCH_OR_RETURN(launch_pdl(pack_tiles_kernel, dim3(grid), dim3(256), 0, st,
                                static_cast<const uint8_t *>(src), rows, row_bytes,
                                static_cast<uint8_t *>(dst)));
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_block_quant(const uint16_t *in, int rows, int cols, int ld, int block_rows,
                               int tiled, uint8_t *q, float *scales, cudaStream_t st,
                               int *launches, bool ue8m0) {
    if (rows == 0) return cudaSuccess;
    const int sms = num_sms();
    mark_launch(st, *launches, block_rows == 1 ? "quant_1x128" : "quant_128x128");
    if (block_rows == 1) {
        const long long total = static_cast<long long>(rows) * (cols / 8);
        const long long want = (total + 255) / 256;
        const int grid = static_cast<int>(want < sms * 16LL ? want : sms * 16LL);
        LAUNCH_OR_RETURN(launch_pdl(quant_1x128_kernel, dim3(grid), dim3(256), 0, st, in, rows, cols, ld, q,
                                    scales, ue8m0 ? 1 : 0));
    } else {
        const long long nblocks = static_cast<long long>(cols / 128) * ((rows + 127) / 128);
        const int grid = static_cast<int>(nblocks < sms * 8LL ? nblocks : sms * 8LL);
        LAUNCH_OR_RETURN(launch_pdl(quant_128x128_kernel, dim3(grid), dim3(256), 0, st, in, rows, cols, ld,
                                    tiled, q, scales, ue8m0 ? 1 : 0));
    }
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_rstd(const uint16_t *h, int T, int d, float eps, float *rstd, cudaStream_t st,
                        int *launches) {
    mark_launch(st, *launches, "prenorm_rstd");
    LAUNCH_OR_RETURN(launch_pdl(rstd_kernel, dim3((T + 7) / 8), dim3(256), 0, st, h, T, d, eps, rstd));
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_quant_scatter(const uint16_t *x, int T, int d, int k, int n_shared,
                                 const int32_t *row_of, uint8_t *a, float *a_scales,
                                 cudaStream_t st, int *launches, PreNorm pn, bool ue8m0) {
    mark_launch(st, *launches, "quant_scatter");
    LAUNCH_OR_RETURN(launch_pdl(quant_scatter_kernel, dim3(T, (d / 128 + 15) / 16), dim3(256), 0, st, x, T, d, k, n_shared, row_of,
                                a, a_scales, pn, ue8m0 ? 1 : 0));
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_scatter_bf16(const uint16_t *x, int T, int d, int k, int n_shared,
                                const int32_t *row_of, uint16_t *a, cudaStream_t st,
                                int *launches, PreNorm pn) {
    mark_launch(st, *launches, "scatter_bf16");
    LAUNCH_OR_RETURN(launch_pdl(scatter_bf16_kernel, dim3(T, (d / 8 + 255) / 256), dim3(256), 0, st, x, T, d, k, n_shared, row_of,
                                a, pn));
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
