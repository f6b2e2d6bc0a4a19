// Internal launchers of the MoE layer library (host side of each kernel
// file).  Each returns the launch error, if any, and adds the number of
// kernels it enqueued to *launches.
#pragma once

#include <atomic>

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/moe_fwd.h"

#include <utility>

namespace moe {

// Launch with programmatic dependent launch allowed: the kernel may start
// while its predecessor on the stream finishes; every kernel of this library
// calls pdl_wait() (griddepcontrol.wait) before it reads anything an earlier
// launch wrote, so only its prologue overlaps the predecessor's tail.
#define LAUNCH_OR_RETURN(call)                 \
    do {                                       \
        const cudaError_t e_l_ = (call);       \
        if (e_l_ != cudaSuccess) return e_l_;  \
    } while (0)

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

constexpr int kTileM = 128;  // rows per grouped-GEMM tile (tcgen05 M)

// Scratch of the permutation and of the grouped GEMM's tile table.
struct PermScratch {
    uint32_t *masks;     // [nblk][E][8] token bit matrix per 256-token block
    int32_t *hist;       // [nblk][E]
    int32_t *blkoff;     // [nblk][E]
    int32_t *seg_start;  // [E + 1] first row of segment s (shared segment last)
    int32_t *seg_rows;   // [E + 1] rows of segment s
    int32_t *tile_start; // [E + 2] prefix of tile_m-row tiles per segment
    int tile_m;          // rows per grouped-GEMM tile: 128, or 64 (64-row MMA tiles)
};

// Pre-norm of the FFN input applied on the fly by the kernels that read it:
// x = bf16((h * rstd[t]) * gamma); rstd == nullptr means the input is x itself.
struct PreNorm {
    const float *rstd;      // [T], from launch_rstd
    const uint16_t *gamma;  // [d] bf16
};

// rstd[t] = 1 / sqrt(sum_i h[t,i]^2 / d + eps), fixed summation order.
cudaError_t launch_rstd(const uint16_t *h, int T, int d, float eps, float *rstd, cudaStream_t st,
                        int *launches);

cudaError_t launch_router(const uint16_t *x, const uint16_t *w, const float *bias, int T, int d,
                          int E, int k, float routed_scale, float *scores, int32_t *idx,
                          float *gates, cudaStream_t st, int *launches, PreNorm pn = {});

cudaError_t launch_permute(const int32_t *idx, int T, int k, int E, int n_shared, PermScratch s,
                           int32_t *counts, int32_t *offsets, int32_t *row_token, int32_t *row_of,
                           int *status, cudaStream_t st, int *launches);

cudaError_t launch_tile_table(const int32_t *offsets, int E, int T, int k, int n_shared,
                              PermScratch s, int *status, cudaStream_t st, int *launches);

// e4m3 quantisation of bf16 [rows, cols] (leading dimension ld) in tiles of
// block_rows x 128.
// ue8m0: power-of-two scales (least 2^k with amax / 2^k <= 448)
cudaError_t launch_block_quant(const uint16_t *in, int rows, int cols, int ld, int block_rows,
                               int tiled, uint8_t *q, float *scales, cudaStream_t st,
                               int *launches, bool ue8m0 = false);

// Row-major [rows, row_bytes] -> 128 x 128-byte tiles (MOE_LAYOUT_TILED).
cudaError_t launch_pack_tiles(const void *src, int rows, int row_bytes, void *dst, cudaStream_t st,
                              int *launches);

// Quantise each token row of x once (1x128 tiles) and write its codes and
// scales to its k routed rows (row_of) and, with n_shared, to row T*k + t.
cudaError_t launch_quant_scatter(const uint16_t *x, int T, int d, int k, int n_shared,
                                 const int32_t *row_of, uint8_t *a, float *a_scales,
                                 cudaStream_t st, int *launches, PreNorm pn = {},
                                 bool ue8m0 = false);

// bf16 copy of each token row to its k routed rows and its shared row.
cudaError_t launch_scatter_bf16(const uint16_t *x, int T, int d, int k, int n_shared,
                                const int32_t *row_of, uint16_t *a, cudaStream_t st,
                                int *launches, PreNorm pn = {});

// residual (nullable, bf16 [T, d]) is added before the final rounding.
cudaError_t launch_combine(const uint16_t *y, const int32_t *row_of, const float *gates, int T,
                           int d, int k, int n_shared, uint16_t *out, cudaStream_t st,
                           int *launches, const uint16_t *residual = nullptr);

// Grouped GEMM over the segment table.
//   gate_up = true : out = H [rows, N_out] = silu(A Wg^T) * (A Wu^T), B rows per
//                    slot = 2*N_out (gate rows then up rows); fp8: H quantised
//                    1x128 with scales h_scales [rows, N_out/128]; bf16: H bf16
//   gate_up = false: out = Y [rows, N_out] bf16 = A W^T, B rows per slot N_out
struct GemmArgs {
    bool fp8;
    bool gate_up;
    const void *a;          // [rows_total, K]
    const float *a_scales;  // [rows_total, K/128] (fp8)
    const void *b;          // [n_slots, B rows, K]: 128 x 128-byte tiles, or row-major
    bool b_rowmajor;        // b (and its layout) row-major instead of tiled
    // expert parallelism (see KParams): per-segment weight slot, and the
    // return of Y rows to the source ranks' buffers (seg_ret NULL: none)
    const int32_t *seg_slot = nullptr, *seg_src = nullptr, *seg_ret = nullptr;
    uint16_t *const *ret_y_dev = nullptr;  // device array: each source rank's Y buffer
    const float *b_scales;  // [n_slots, B rows/128, K/128] (fp8)
    void *out;              // H or Y
    float *out_scales;      // H scales (fp8 gate_up)
    int rows_total;         // R_s
    int K;
    int N_out;
    int n_slots;
    int n_segments;         // E + n_shared
    int E;                  // segments 0..E-1 use slot s; segment E uses slot E
    const int32_t *seg_start, *seg_rows, *tile_start;
    int *status;
    int inject_fault;       // test hook: make one bounded wait run out (see api.cu)
    bool ue8m0;             // fp8 gate/up: H requantised with power-of-two scales
    int tile_m;             // rows per tile of the segment table (64: M=64 MMA tiles, fp32 scales)
    // seg_start == nullptr: one segment of all rows_total rows (no table)
    // Split K of the down GEMM (fp32-scale and bf16 paths): ksplit > 1 work
    // items per output tile over consecutive K ranges write binary32 partial
    // sums to partial [ksplit][rows_total][N_out] instead of Y; the caller
    // then runs launch_splitk_reduce.
    int ksplit;
    float *partial;
    const uint16_t *residual;  // down GEMM without split: bf16 [rows_total, N_out] added before rounding
};
constexpr int kMaxSplitK = 8;
constexpr int kMaxEpRanks = MOE_EP_MAX_RANKS;  // ranks of an expert-parallel group
// Output tiles of a GEMM with one segment of `rows` rows.
inline int gemm_output_tiles(int rows, int N_out) { return ((rows + 127) / 128) * (N_out / 256); }
// out [rows, n] = bf16(sum of the ksplit partial sums in order (+ residual)).
cudaError_t launch_splitk_reduce(const float *partial, int ksplit, int rows, int n,
                                 const uint16_t *residual, uint16_t *out, cudaStream_t st,
                                 int *launches);
cudaError_t launch_grouped_gemm(const GemmArgs &g, cudaStream_t st, int *launches);

int num_sms();

// Unique id of the calling thread's current CUDA context, or 0 if there is
// none or the driver cannot tell (api.cu).  Ids are never reused within a
// process, unlike context handles.
unsigned long long current_context_id();

// Function attributes (dynamic shared memory size) belong to the module
// loaded in a device's context, so they are set again whenever the context
// changes (a device reset destroys the primary context and its modules).
// One flag word per call site: the context id each device was configured in
// (devices 0..63; larger device numbers, and a driver that reports no ids,
// are configured on every call).
struct DeviceConfigured {
    std::atomic<unsigned long long> ctx[64];
};
inline bool first_use_on_device(DeviceConfigured &done) {
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long id = current_context_id();
    if (dev < 0 || dev >= 64 || id == 0) return true;
    return done.ctx[dev].load(std::memory_order_acquire) != id;
}
inline void mark_used_on_device(DeviceConfigured &done) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64) done.ctx[dev].store(current_context_id(), std::memory_order_release);
}

// Error/launch bookkeeping shared by the C entry points (api.cu).
// Expert parallelism: the segment table of a grouped GEMM over received rows.
struct EpTableArgs {
    const int32_t *start, *rows, *slot, *src, *ret;  // device arrays [n_seg]; slot may be NULL
    int n_seg, rows_total, n_slots, world, tile_m;
    int ret_capacity[kMaxEpRanks];  // rows of each source rank's Y buffer
    uint16_t *ret_y[kMaxEpRanks];   // each source rank's Y buffer
};
// Also writes a.ret_y to ret_y_dev [world] (device memory the GEMM reads).
cudaError_t launch_ep_table(const EpTableArgs &a, int32_t *seg_start, int32_t *seg_rows,
                            int32_t *tile_start, int32_t *seg_slot, int32_t *seg_src,
                            int32_t *seg_ret, uint16_t **ret_y_dev, int *status, cudaStream_t st,
                            int *launches);

// Expert parallelism: rows of one source rank's permuted buffer copied into
// the owners' receive buffers, one contiguous block per owner.
struct EpDispatchArgs {
    int n_blocks, row_bytes, n_scales;
    int src_row[kMaxEpRanks], dst[kMaxEpRanks], dst_row[kMaxEpRanks];
    int prefix[kMaxEpRanks + 1];  // rows of blocks before block b
    uint8_t *dst_a[kMaxEpRanks];
    float *dst_s[kMaxEpRanks];
};
cudaError_t launch_ep_dispatch(const void *a, const float *a_scales, const EpDispatchArgs &g,
                               cudaStream_t st, int *launches);

int record_error(int code, const char *msg);  // sets moe_last_error, returns code
void record_launches(int n);                   // sets moe_last_launch_count
int validate_shape(const moe_shape *s);        // host-side shape checks
int validate_device();                         // MOE_ERR_UNSUPPORTED unless the device is sm_100

// Called just before the call's kernel launch number `index` with that
// kernel's name (and once more after the last launch, without a name):
// records the caller's event `index` on `st` when the moe_set_kernel_events
// hook is active, and the name for moe_last_launch_name.
void mark_launch(cudaStream_t st, int index, const char *name = nullptr);

// NVTX range of one library call on the calling thread (the per-kernel ranges
// that mark_launch opens nest inside it); closes them on every return path.
struct CallRange {
    explicit CallRange(const char *name);
    ~CallRange();
    CallRange(const CallRange &) = delete;
    CallRange &operator=(const CallRange &) = delete;
};

}  // namespace moe
