/*
 * moe_fwd.h — C ABI of the B200 (sm_100a) forward pass of one
 * DeepSeek-V3/R1 Mixture-of-Experts FFN layer.
 *
 * The layer (sources are the pages' titles and sections):
 *  - "DeepSeek-R1" architecture card (llm-architectures-explained.vercel.app),
 *    table "Every architecture field": d_model 7168, 256 routed experts,
 *    8 active per token, gated experts of width 2048, 1 shared expert.
 *  - "DeepSeek v3 and R1 Model Architecture" (onlylabs.fyi), section "Local
 *    Balanced Routing to Experts": tokens go to experts by token-to-expert
 *    affinity; a per-expert bias is added for routing only.  Section
 *    "Structural change": the shared expert is always active.
 *  - "DeepSeek-R1" (aguasto.com), section "Quantization": blockwise FP8.
 * Readings where the pages are silent: affinity s = sigmoid(l) on binary32
 * logits accumulated by sequential fused multiply-adds over d_model; top-k
 * by (s + bias) descending, lowest expert index first among equals; gates
 * g = s / sum(selected s) * routed_scale; the shared expert has weight 1;
 * FP8 is OCP e4m3 with 1x128 activation tiles and 128x128 weight blocks,
 * each with a binary32 scale amax/448, and the expert GEMMs accumulate each
 * 128-wide K block separately, then scale it and add it in binary32.
 *
 * Conventions for every call:
 *  - Every pointer is caller-owned DEVICE memory unless stated otherwise; the
 *    library never allocates or frees device memory.
 *  - "bf16" buffers hold bfloat16 bit patterns (uint16_t); "e4m3" buffers
 *    hold OCP FP8 E4M3 codes (uint8_t).  Matrices are row-major, contiguous.
 *  - Device pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *  - `stream` is a cudaStream_t (NULL: the legacy default stream).  Calls are
 *    asynchronous: they only enqueue kernels.  Arguments are read by the
 *    kernels when they run, so buffers must stay valid until then.
 *  - Return value: MOE_OK, or a negative MOE_ERR_* code, in which case no
 *    kernel was enqueued (except MOE_ERR_CUDA, raised when a launch failed).
 *    moe_last_error() gives a message for the calling thread's last error.
 *  - Errors found by the kernels themselves (an expert index out of range,
 *    a duplicate expert for one token, a bounded device wait that ran out)
 *    are recorded in a status word at the start of the workspace; read and
 *    clear it with moe_check_status().  A kernel that records an error skips
 *    the offending access and finishes, so the CUDA context stays usable.
 *  - The library keeps per-device state (kernel attributes, the no-alloc
 *    router's scratch address) keyed by the device's current context, so it
 *    keeps working after the device is reset (cudaDeviceReset) and its
 *    context created again.
 *  - Shapes: d_model a multiple of 256, d_expert a multiple of 128;
 *    1 <= top_k <= min(n_experts, 32); n_shared 0 or 1; n_experts + n_shared
 *    <= 1024; T >= 0 (T = 0 enqueues nothing).
 */
#ifndef MOE_FWD_H
#define MOE_FWD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1, /* null/misaligned pointer, bad shape value     */
    MOE_ERR_UNSUPPORTED = -2, /* valid but not implemented (e.g. no sm_100a)  */
    MOE_ERR_WORKSPACE = -3,   /* workspace smaller than moe_workspace_size()  */
    MOE_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed         */
    MOE_ERR_TIMEOUT = -5,     /* a bounded device-side wait ran out           */
    MOE_ERR_DEVICE_INDEX = -6 /* kernel saw an expert index out of range or a
                                 token that selected one expert twice        */
};

enum moe_precision {
    MOE_BF16 = 0,      /* bf16 weights and activations, binary32 accumulate */
    MOE_FP8_BLOCK = 1, /* e4m3 1x128 activations, 128x128 weights, fp32 scales */
    MOE_FP8_UE8M0 = 2  /* as MOE_FP8_BLOCK with power-of-two scales (UE8M0 values
                          stored as fp32); see fp8_block_quant_ue8m0 */
};

/* Weight storage (moe_shape.weight_layout, moe_dense_shape.weight_layout).
 * The expert GEMMs read their weights in either of two layouts:
 *  - MOE_LAYOUT_ROWMAJOR: each expert matrix [N, K] row-major, contiguous,
 *    experts stacked ([n, N, K]); the layout of the problem statement.
 *  - MOE_LAYOUT_TILED: a row-major matrix of R rows x C bytes (R, C
 *    multiples of 128) stored as (R/128) x (C/128) tiles of 128 rows x 128
 *    bytes, tile (i, j) at byte offset (i * (C/128) + j) * 16384, row r of a
 *    tile at r * 128 inside it.  For a stack [n, N, K] of expert matrices,
 *    R = n*N.  Each tile is one contiguous 16 KB read (for e4m3 exactly one
 *    128x128 scale block), which the small (weight-streaming) batches read
 *    at full HBM bandwidth.
 * The layout of the weights a call reads is the one its shape declares; a
 * zero-initialised shape declares MOE_LAYOUT_ROWMAJOR.  Scales are [n,
 * N/128, K/128] row-major in both. */
enum moe_layout {
    MOE_LAYOUT_ROWMAJOR = 0,
    MOE_LAYOUT_TILED = 1
};

/* Layer shape.  T tokens, d_model, n_experts routed experts (E), top_k (k),
 * d_expert, n_shared (0 or 1 shared experts of width d_expert),
 * routed_scale (multiplies every gate), precision (enum moe_precision),
 * weight_layout (enum moe_layout) of w13 and w2; any other value is
 * rejected with MOE_ERR_INVALID_ARG. */
typedef struct moe_shape {
    int T;
    int d_model;
    int n_experts;
    int top_k;
    int d_expert;
    int n_shared;
    float routed_scale;
    int precision;
    int weight_layout;
} moe_shape;

/* Bytes of device workspace that moe_forward needs for this shape (the other
 * calls need no more).  0 if the shape is invalid (see moe_last_error). */
size_t moe_workspace_size(const moe_shape *shape);

/* Where moe_forward / moe_forward_prenorm keep their intermediate results
 * inside the workspace: byte offsets from its start, for inspection (tests,
 * debugging).  Once the call's kernels have run, the regions hold
 *   scores    fp32 [T, n_experts]  affinities s = sigmoid(l)
 *   topk_idx  int32 [T, top_k]     (only when topk_idx_out was NULL)
 *   topk_w    fp32 [T, top_k]      gates
 *   counts, offsets, row_token, row_of   the permutation (as moe_permute)
 *   a         [R_s, d_model] e4m3 (fp8 precisions) or bf16: permuted rows of x
 *   a_scales  fp32 [R_s, d_model/128] (fp8 precisions)
 *   h, h_scales   [R_s, d_expert] H (e4m3 + scales, or bf16)
 *   y         bf16 [R_s, d_model]  expert outputs before the combine
 * with R_s = T*(top_k + n_shared).  The layout is fixed by the shape.
 * Returns MOE_OK, or MOE_ERR_INVALID_ARG (invalid shape, NULL out). */
typedef struct moe_workspace_offsets {
    size_t status, scores, topk_idx, topk_w, counts, offsets, row_token, row_of;
    size_t a, a_scales, h, h_scales, y, total;
} moe_workspace_offsets;
int moe_workspace_layout(const moe_shape *shape, moe_workspace_offsets *out);

/* Router: logits l = x W_r^T in binary32 (sequential fused multiply-adds over
 * d_model), affinity s = sigmoid(l), selection by s + bias (bias: routing
 * only), top-k in rank order, gates g_j = s_j / sum_selected(s) *
 * routed_scale ("Local Balanced Routing to Experts").
 *   x        bf16 [T, d_model]
 *   w_router bf16 [n_experts, d_model]
 *   bias     fp32 [n_experts]
 *   topk_idx int32 [T, top_k] out: expert ids, best first
 *   topk_w   fp32 [T, top_k]  out: gates in the same order
 *   ws       workspace (>= moe_workspace_size bytes): holds the [T, E] scores
 * When the scores kernel's grid fits in one wave, its blocks ask for unused
 * shared memory so that no SM holds more of them than the wave needs; a
 * kernel that the caller runs concurrently on another stream then finds less
 * shared memory free on those SMs for the scores kernel's duration. */
int moe_route(const moe_shape *shape, const uint16_t *x, const uint16_t *w_router,
              const float *bias, int32_t *topk_idx, float *topk_w,
              void *ws, size_t ws_bytes, void *stream);

/* Router for callers that cannot allocate device memory.  The pages have no
 * counterpart to this call: it exists for callers that are not allowed to call
 * cudaMalloc and have no workspace to pass, e.g. code inside a host
 * framework's plugin interface that owns all device memory, or a serving loop
 * that forbids allocation after start-up because cudaMalloc can synchronise
 * the device and stall every other stream.  Same computation and outputs as
 * moe_route, but its [T, E] score scratch is a fixed array inside the library
 * (MOE_ROUTE_NOALLOC_MAX_SCORES floats, 4 MiB, held on every GPU that loads
 * the library until the process exits).
 *   - T * n_experts above MOE_ROUTE_NOALLOC_MAX_SCORES: MOE_ERR_INVALID_ARG,
 *     nothing enqueued.
 *   - The first call on a device looks up the array's device address (with
 *     that device current), so make that first call before any stream capture.
 *     The address is looked up again when the device's context has changed
 *     (after cudaDeviceReset, the library's module is loaded anew), so the
 *     first call after a reset should also come before any stream capture.
 *   - Error codes as moe_route (MOE_ERR_UNSUPPORTED on a device that is not
 *     sm_100).
 *   - Every call shares the one array: calls whose kernels overlap on the GPU
 *     (other streams, other host threads) race and must be serialised by the
 *     caller.  The array keeps the last call's scores; nothing in it needs to
 *     start at zero.
 *   - Allocates nothing (no cudaMalloc/cudaFree, no allocating library call). */
#define MOE_ROUTE_NOALLOC_MAX_SCORES (1 << 20)
int moe_route_noalloc(const moe_shape *shape, const uint16_t *x, const uint16_t *w_router,
                      const float *bias, int32_t *topk_idx, float *topk_w, void *stream);

/* Permutation into per-expert segments (expert order; tokens ascending inside
 * a segment; deterministic).
 *   topk_idx  int32 [T, top_k] in
 *   counts    int32 [n_experts] out: tokens per expert
 *   offsets   int32 [n_experts + 1] out: exclusive prefix sum, offsets[E] = T*k
 *   row_token int32 [T*k] out: token of each routed row
 *   row_of    int32 [T, top_k] out: routed row of (t, topk_idx[t, j])
 * The shared segment is implicit: rows T*k .. T*k+T-1 hold tokens 0..T-1. */
int moe_permute(const moe_shape *shape, const int32_t *topk_idx, int32_t *counts,
                int32_t *offsets, int32_t *row_token, int32_t *row_of,
                void *ws, size_t ws_bytes, void *stream);

/* Blockwise e4m3 quantisation ("Quantization": blockwise FP8) of a bf16
 * [rows, cols] matrix with leading dimension ld (elements, >= cols, multiple
 * of 8).  Tiles are block_rows x 128 (block_rows 1 for activations, 128 for
 * weights; a short last row block is allowed in row-major output).  Per tile
 * amax; scale = amax / 448, codes = e4m3_rn_satfinite(v * (448 / amax)); an
 * all-zero tile gets scale 1 and +0 codes.
 *   out_layout MOE_LAYOUT_ROWMAJOR: q is e4m3 [rows, cols] (leading dimension
 *              cols); MOE_LAYOUT_TILED (block_rows 128, rows % 128 == 0):
 *              q holds the same codes in the tiled layout the GEMMs read
 *   scales fp32 [ceil(rows / block_rows), cols / 128] out
 * A stack of expert matrices [n, N, K] with N % 128 == 0 is one call with
 * rows = n*N, cols = K. */
int fp8_block_quant(const uint16_t *in, int rows, int cols, int ld, int block_rows,
                    int out_layout, uint8_t *q, float *scales, void *stream);

/* The same quantisation with power-of-two scales (the UE8M0 variant used by
 * MOE_FP8_UE8M0; the pages give blockwise FP8 with per-block scales, the
 * power-of-two rounding is this library's reading of the variant): per tile
 * scale = 2^k for the least integer k >= -127 with amax / 2^k <= 448 (an
 * all-zero tile: 2^0), codes = e4m3_rn(v * 2^-k), the multiply being exact
 * and never saturating.  Arguments, layouts and errors as fp8_block_quant;
 * the scales are written as fp32 values (each exactly 2^k). */
int fp8_block_quant_ue8m0(const uint16_t *in, int rows, int cols, int ld, int block_rows,
                          int out_layout, uint8_t *q, float *scales, void *stream);

/* Repacks a row-major matrix of `rows` rows x `row_bytes` bytes (both
 * multiples of 128; src and dst 16-byte aligned, not overlapping) into the
 * tiled layout (MOE_LAYOUT_TILED).  Used once, ahead of time, for bf16
 * expert weights; pure data movement. */
int moe_pack_tiles(const void *src, int rows, int row_bytes, void *dst, void *stream);

/* Grouped gated expert MLP over the permuted rows (card: "experts are gated
 * MLPs"): for every segment s (routed experts 0..E-1, then the shared expert
 * at slot E when n_shared = 1)  H = silu(A_s W_gate,s^T) * (A_s W_up,s^T),
 * Y_s = H W_down,s^T.  R_s = T*k + T*n_shared rows.
 *   a          [R_s, d_model] bf16, or e4m3 codes in MOE_FP8_BLOCK / _UE8M0
 *   a_scales   fp32 [R_s, d_model/128] (fp8 precisions) or NULL
 *   offsets    int32 [n_experts + 1] segment starts (as from moe_permute)
 *   w13        [E + n_shared, 2*d_expert, d_model]: gate rows, then up rows,
 *              e4m3 or bf16, in the shape's weight_layout
 *   w13_scales fp32 [E + n_shared, 2*d_expert/128, d_model/128] or NULL
 *   w2         [E + n_shared, d_model, d_expert], in the shape's weight_layout
 *   w2_scales  fp32 [E + n_shared, d_model/128, d_expert/128] or NULL
 *   y          bf16 [R_s, d_model] out
 * In MOE_FP8_BLOCK, H is quantised 1x128 (e4m3) before the down GEMM (with
 * power-of-two scales in MOE_FP8_UE8M0); in MOE_BF16 it is rounded to bf16.
 * Accumulation is binary32. */
int moe_grouped_swiglu(const moe_shape *shape, const void *a, const float *a_scales,
                       const int32_t *offsets, const void *w13, const float *w13_scales,
                       const void *w2, const float *w2_scales, uint16_t *y,
                       void *ws, size_t ws_bytes, void *stream);

/* Quantise-and-scatter, the step between moe_permute and the grouped GEMMs
 * ("DeepSeek-R1", "Quantization": blockwise FP8 with 1x128 activation
 * tiles): row row_of[t, j] of `a` receives token t's codes for its j-th
 * expert, and row T*k + t the shared expert's copy (n_shared = 1); in the
 * fp8 precisions each row is x[t] quantised 1x128 (scale amax/448, or the
 * power-of-two scale in MOE_FP8_UE8M0), in MOE_BF16 it is x[t] itself.
 *   x        bf16 [T, d_model]; row_of int32 [T, top_k] (from moe_permute)
 *   a        [R_s, d_model] e4m3 codes (fp8 precisions) or bf16 out
 *   a_scales fp32 [R_s, d_model/128] out (fp8 precisions; NULL in MOE_BF16)
 * R_s = T*(top_k + n_shared).  The same kernel moe_forward runs. */
int moe_quant_scatter(const moe_shape *shape, const uint16_t *x, const int32_t *row_of, void *a,
                      float *a_scales, void *stream);

/* Weighted un-permute plus the always-on shared expert ("Structural change":
 * an always-activated expert): out[t] = bf16( sum_j topk_w[t,j] *
 * y[row_of[t,j]] + y[T*k + t] ), binary32 accumulation in rank order (the
 * shared term only when n_shared = 1).
 *   y bf16 [R_s, d_model]; row_of int32 [T, k]; topk_w fp32 [T, k];
 *   out bf16 [T, d_model] */
int moe_combine(const moe_shape *shape, const uint16_t *y, const int32_t *row_of,
                const float *topk_w, uint16_t *out, void *stream);

/* The whole layer: route, permute, quantise-and-scatter (or bf16 scatter),
 * grouped gate/up GEMM + SwiGLU, grouped down GEMM, combine.
 *   x [T, d_model] bf16 in; out [T, d_model] bf16 out.
 *   w13/w2 and scales as for moe_grouped_swiglu, in the shape's
 *   weight_layout (e4m3 weights are quantised once, ahead of time, with
 *   fp8_block_quant in MOE_FP8_BLOCK or fp8_block_quant_ue8m0 in
 *   MOE_FP8_UE8M0, with out_layout = the shape's weight_layout; bf16
 *   weights are used as they are, or repacked once with moe_pack_tiles for
 *   MOE_LAYOUT_TILED).
 *   topk_idx_out int32 [T, k] or NULL: receives the routing decision. */
int moe_forward(const moe_shape *shape, const uint16_t *x, const uint16_t *w_router,
                const float *bias, const void *w13, const float *w13_scales,
                const void *w2, const float *w2_scales, uint16_t *out,
                int32_t *topk_idx_out, void *ws, size_t ws_bytes, void *stream);

/* The FFN block around the layer ("DeepSeek-R1" card, "Facts": pre-norm,
 * RMSNorm before the MLP): out = h + MoE(x) with x = bf16((h * rstd) *
 * gamma), rstd = 1 / sqrt(sum_i h_i^2 / d_model + eps).  x is never written:
 * the router and the quantise/scatter step normalise h as they read it, and
 * the combine adds h before its final rounding.  sum_i h_i^2 is binary32 in
 * a fixed order (32 lane sums over i mod 32, fused multiply-add in ascending
 * i, then xor-butterfly pairwise adds), so routing stays reproducible.
 *   h     bf16 [T, d_model] (the residual stream)
 *   gamma bf16 [d_model]; eps >= 0 (DeepSeek-V3 uses 1e-6)
 *   other arguments as for moe_forward. */
int moe_forward_prenorm(const moe_shape *shape, const uint16_t *h, const uint16_t *gamma,
                        float eps, const uint16_t *w_router, const float *bias, const void *w13,
                        const float *w13_scales, const void *w2, const float *w2_scales,
                        uint16_t *out, int32_t *topk_idx_out, void *ws, size_t ws_bytes,
                        void *stream);

/* ------------------------------------------------------------------------
 * Dense FFN layer: the first layers of the model, before the MoE layers
 * ("DeepSeek-R1" architecture card, "Every architecture field": layout
 * 3 x dense then 58 x MoE; ffns.dense is a gated MLP with d_ff 18432).
 *   out = H W2^T,  H = silu(x Wg^T) * (x Wu^T)
 * computed on the same kernels as the experts, with the same numerics per
 * precision (x quantised 1x128, weights 128x128, H requantised 1x128 before
 * the down GEMM; bf16: H rounded to bf16), every row of x in one segment.
 * Shapes: d_model a multiple of 256, d_ff a multiple of 128, T >= 0. */
typedef struct {
    int T;             /* tokens */
    int d_model;       /* 7168 for DeepSeek-V3 */
    int d_ff;          /* 18432 for DeepSeek-V3 */
    int precision;     /* enum moe_precision */
    int weight_layout; /* enum moe_layout of w13 and w2 */
} moe_dense_shape;

/* Bytes of workspace moe_dense_ffn needs (0 on an invalid shape).  It holds
 * the status word first (read with moe_check_status), the quantised x, H,
 * and for small batches the split-K partial sums of the down GEMM. */
size_t moe_dense_workspace_size(const moe_dense_shape *shape);

/* The dense layer.
 *   x   bf16 [T, d_model]; out bf16 [T, d_model]: Y rounded once to bf16,
 *       stored by the down GEMM, or (batches of at most 256 tokens, whose
 *       down GEMM splits K over the SMs) by a kernel that adds the K ranges'
 *       binary32 partial sums in order, so results do not depend on timing
 *   w13 [2*d_ff, d_model] (gate rows, then up rows) and w2 [d_model, d_ff]
 *       in the shape's weight_layout, e4m3 with scales [2*d_ff/128, d_model/128] and
 *       [d_model/128, d_ff/128] (MOE_FP8_BLOCK / MOE_FP8_UE8M0), or bf16
 *       with NULL scales (MOE_BF16): the layout of one expert slot.
 *   ws: moe_dense_workspace_size bytes, zero-filled once before first use. */
int moe_dense_ffn(const moe_dense_shape *shape, const uint16_t *x, const void *w13,
                  const float *w13_scales, const void *w2, const float *w2_scales,
                  uint16_t *out, void *ws, size_t ws_bytes, void *stream);

/* The dense FFN block with its pre-norm and residual: out = bf16(h + FFN(x))
 * with x = bf16((h * rstd) * gamma) as in moe_forward_prenorm; the residual
 * is added to the binary32 down-GEMM sum before its one rounding (Y is not
 * stored). */
int moe_dense_ffn_prenorm(const moe_dense_shape *shape, const uint16_t *h,
                          const uint16_t *gamma, float eps, const void *w13,
                          const float *w13_scales, const void *w2, const float *w2_scales,
                          uint16_t *out, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Expert parallelism ("DeepSeek v3 and R1 Model Architecture", "Local
 * Balanced Routing to Experts": routed experts are spread over devices,
 * tokens travel to the devices that hold their experts, and the routing
 * keeps the load of devices and of communication balanced).
 * G ranks; rank r owns routed experts r*P .. r*P + P - 1 (P = n_experts / G);
 * every rank holds the shared expert.  One layer call:
 *  1. every rank, on its own tokens: moe_route, moe_permute,
 *     moe_quant_scatter.  Its routed rows are in global expert order, so its
 *     rows for owner o form one contiguous block;
 *  2. the ranks exchange their per-expert counts and derive the exchange
 *     plan (which block goes where; the segments of each owner's receive
 *     buffer; where results return);
 *  3. every rank (a source): moe_ep_dispatch copies its block for each owner
 *     into that owner's receive buffer;
 *  4. every rank (an owner): moe_ep_grouped_swiglu over its received rows,
 *     one segment per (source, local expert); the down GEMM's epilogue
 *     stores each Y row straight into its source's Y buffer, at the row's
 *     place in the source's permuted order;
 *  5. every rank: moe_ep_grouped_swiglu over its own shared rows (one
 *     segment, the shared expert's weights, returning into its own Y
 *     buffer), then moe_combine.
 * Destination pointers may be other GPUs' memory (peer mappings) or, for
 * ranks emulated on one GPU, buffers of this one; the kernels only load this
 * GPU's memory (no TMA multicast) and store with plain stores. */
#define MOE_EP_MAX_RANKS 64

/* One contiguous block of a source's rows for one owner. */
typedef struct moe_ep_block {
    int src_row;  /* first row in the source's permuted buffer `a` */
    int rows;     /* rows in the block (0: nothing to send) */
    int dst;      /* owner rank (index into recv_a / recv_scales) */
    int dst_row;  /* first row in the owner's receive buffer */
} moe_ep_block;

/* Dispatch (step 3): copies each block's rows of `a` (and their fp32 block
 * scales in the fp8 precisions) into recv_a[dst] / recv_scales[dst].
 *   a          [a_rows, d_model] e4m3 or bf16 (from moe_quant_scatter)
 *   a_scales   fp32 [a_rows, d_model/128] (fp8 precisions) or NULL
 *   blocks     host array of n_blocks (0..MOE_EP_MAX_RANKS) blocks
 *   recv_a, recv_scales, recv_capacity  host arrays of `world` entries:
 *              device pointers of each owner's receive buffer ([capacity,
 *              d_model] codes, [capacity, d_model/128] scales) and its rows
 * Every block is checked on the host against a_rows and the destination's
 * capacity (MOE_ERR_INVALID_ARG otherwise, nothing enqueued).  Blocks must
 * not overlap in a destination.  Reads only shape->d_model and precision. */
int moe_ep_dispatch(const moe_shape *shape, const void *a, const float *a_scales, int a_rows,
                    int n_blocks, const moe_ep_block *blocks, int world, void *const *recv_a,
                    float *const *recv_scales, const int *recv_capacity, void *stream);

/* Bytes of workspace moe_ep_grouped_swiglu needs for `rows` received rows in
 * n_segments (1..1024) segments (0 if invalid): the status word first, the
 * checked segment table, H and its scales. */
size_t moe_ep_workspace_size(const moe_shape *shape, int rows, int n_segments);

/* The owner's grouped gated MLP over received rows (step 4), or a rank's
 * shared expert over its own shared rows (step 5): for segment i (rows
 * seg_start[i] .. + seg_rows[i] of `a`, weight slot seg_slot[i], or i when
 * seg_slot is NULL)  H = silu(A W_gate^T) * (A W_up^T),  Y = H W_down^T,
 * numerics as moe_grouped_swiglu (H requantised 1x128 in the fp8
 * precisions).  Row j of segment i is stored in ret_y[seg_src[i]] at row
 * seg_ret[i] + (j - seg_start[i]) (bf16 [.., d_model]).
 *   a, a_scales     [rows, d_model] received rows (e4m3 + fp32 scales, or bf16)
 *   seg_*           int32 device arrays [n_segments]
 *   w13, w2, scales n_slots weight slots laid out as for moe_grouped_swiglu
 *                   (gate rows then up rows), in the shape's weight_layout
 *   ret_y, ret_capacity  host arrays of `world` entries: each source's Y
 *                   buffer (device pointer; may be NULL when its capacity is
 *                   0) and its rows
 * Segments that reach outside `a`, name a slot or source that does not
 * exist, or would store past a source's capacity are recorded in the
 * status word (MOE_ERR_DEVICE_INDEX, read with moe_check_status) and
 * skipped.  Reads shape->d_model, d_expert, precision and weight_layout. */
int moe_ep_grouped_swiglu(const moe_shape *shape, int rows, const void *a, const float *a_scales,
                          int n_segments, const int32_t *seg_start, const int32_t *seg_rows,
                          const int32_t *seg_slot, const int32_t *seg_src, const int32_t *seg_ret,
                          int n_slots, const void *w13, const float *w13_scales, const void *w2,
                          const float *w2_scales, int world, uint16_t *const *ret_y,
                          const int *ret_capacity, void *ws, size_t ws_bytes, void *stream);

/* Synchronises `stream`, returns the workspace status word (MOE_OK or the
 * first device-recorded MOE_ERR_*), and resets it to MOE_OK.  A workspace must
 * be zero-filled once before first use (or passed here once) so its status
 * word starts clean. */
int moe_check_status(void *ws, void *stream);

/* Message for the calling thread's last failed call ("" if none). */
const char *moe_last_error(void);

/* Number of kernels the last successful call on this thread enqueued. */
int moe_last_launch_count(void);

/* Name of kernel i (0 <= i < moe_last_launch_count()) of the last successful
 * call on this thread, in launch order (for example "router_scores",
 * "perm_small", "grouped_gemm_gate_up"); NULL for any other i.  The string is
 * static: the caller does not free it.  No counterpart in the pages: it lets
 * a profiler attach the moe_set_kernel_events timeline to kernels. */
const char *moe_last_launch_name(int i);

/* Profiling hook.  events: n_events cudaEvent_t handles (host array, owned
 * by the caller) or NULL to switch the hook off.  While set, every later
 * call on this thread records events[i] on its stream just before its i-th
 * kernel launch and events[launches] after the last one (the CUDA-event
 * timeline of each kernel), for indices below n_events; a NULL entry is
 * skipped.  Returns MOE_OK or MOE_ERR_INVALID_ARG. */
int moe_set_kernel_events(void **events, int n_events);

#ifdef __cplusplus
}
#endif

#endif /* MOE_FWD_H */
