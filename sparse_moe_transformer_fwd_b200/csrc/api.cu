// C ABI of the MoE layer library: argument checks, workspace layout and the
// launch order of the forward pass.  See include/moe_fwd.h for the contract.
#include "common.cuh"
#include "kernels.h"

#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

namespace moe {

// Unique id of the calling thread's current CUDA context (driver API, fetched
// through the runtime so the library needs no link-time driver dependency),
// or 0 if there is none or the driver cannot tell.  Ids are never reused in a
// process, unlike context handles: after cudaDeviceReset the new primary
// context may get the old handle.
unsigned long long current_context_id() {
    using GetCurrentFn = int (*)(void **);
    using GetIdFn = int (*)(void *, unsigned long long *);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    void *ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0) return 0;
    return id;
}

int num_sms() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

namespace {
thread_local cudaEvent_t *g_events = nullptr;  // profiling hook (moe_set_kernel_events)
thread_local int g_n_events = 0;
constexpr int kMaxNamed = 64;
thread_local const char *g_names[kMaxNamed];  // kernel of each launch of the last call
thread_local bool g_nvtx_kernel = false;       // a per-kernel NVTX range is open
}  // namespace

void mark_launch(cudaStream_t st, int index, const char *name) {
    if (g_events && index < g_n_events && g_events[index]) cudaEventRecord(g_events[index], st);
    if (name && index >= 0 && index < kMaxNamed) g_names[index] = name;
    // NVTX: one host range per kernel launch, inside the call's range
    if (g_nvtx_kernel) nvtxRangePop();
    g_nvtx_kernel = name != nullptr;
    if (name) nvtxRangePushA(name);
}

CallRange::CallRange(const char *name) { nvtxRangePushA(name); }
CallRange::~CallRange() {
    if (g_nvtx_kernel) nvtxRangePop();
    g_nvtx_kernel = false;
    nvtxRangePop();
}

namespace {

thread_local std::string g_err;
thread_local int g_launches = 0;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *where) {
    return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Fault injection for tests of the bounded device waits, read per call from
// the environment: MOE_FAULT_INJECT=gemm_tx makes the first grouped GEMM of
// the call arm one pipeline stage for bytes that never arrive, so its
// consumer's wait runs out and the call reports MOE_ERR_TIMEOUT through the
// status word (the kernel then drains and exits normally).
bool inject_gemm_fault() {
    const char *v = getenv("MOE_FAULT_INJECT");
    return v && strcmp(v, "gemm_tx") == 0;
}

int check_device() {
    int dev = 0, major = 0, minor = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return fail(MOE_ERR_UNSUPPORTED, "needs an sm_100 device (found sm_%d%d)", major, minor);
    return MOE_OK;
}

int check_shape(const moe_shape *s) {
    if (!s) return fail(MOE_ERR_INVALID_ARG, "shape is NULL");
    if (s->T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
    if (s->d_model <= 0 || s->d_model % 256)
        return fail(MOE_ERR_INVALID_ARG, "d_model must be a positive multiple of 256");
    if (s->d_expert <= 0 || s->d_expert % 128)
        return fail(MOE_ERR_INVALID_ARG, "d_expert must be a positive multiple of 128");
    if (s->n_experts < 1 || s->n_shared < 0 || s->n_shared > 1 ||
        s->n_experts + s->n_shared > 1024)
        return fail(MOE_ERR_INVALID_ARG, "need 1 <= n_experts, n_shared in {0,1}, "
                                         "n_experts + n_shared <= 1024");
    if (s->top_k < 1 || s->top_k > 32 || s->top_k > s->n_experts)
        return fail(MOE_ERR_INVALID_ARG, "need 1 <= top_k <= min(n_experts, 32)");
    if (s->precision != MOE_BF16 && s->precision != MOE_FP8_BLOCK &&
        s->precision != MOE_FP8_UE8M0)
        return fail(MOE_ERR_INVALID_ARG, "unknown precision %d", s->precision);
    if (s->weight_layout != MOE_LAYOUT_ROWMAJOR && s->weight_layout != MOE_LAYOUT_TILED)
        return fail(MOE_ERR_INVALID_ARG, "unknown weight_layout %d", s->weight_layout);
    const long long R_s = static_cast<long long>(s->T) * (s->top_k + s->n_shared);
    if (R_s * s->d_model > (1LL << 40) || R_s > (1LL << 30))
        return fail(MOE_ERR_INVALID_ARG, "T too large");
    return MOE_OK;
}

// e4m3 codes in either scale format (fp32 amax/448 or power-of-two UE8M0)
bool is_fp8(const moe_shape *s) {
    return s->precision == MOE_FP8_BLOCK || s->precision == MOE_FP8_UE8M0;
}
bool is_ue8m0(const moe_shape *s) { return s->precision == MOE_FP8_UE8M0; }

// ---------------------------------------------------------- workspace ---
struct Layout {
    size_t status, rstd, scores, idx, gates, counts, offsets, row_token, row_of;
    size_t masks, hist, blkoff, seg_start, seg_rows, tile_start;
    size_t a, a_scales, h, h_scales, y;
    size_t total;
};

Layout layout(const moe_shape *s) {
    const size_t T = s->T, E = s->n_experts, k = s->top_k, d = s->d_model, de = s->d_expert;
    const size_t Rs = T * (k + s->n_shared);
    const size_t nblk = (T + 255) / 256;
    const bool fp8 = is_fp8(s);
    const size_t es = fp8 ? 1 : 2;
    Layout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~static_cast<size_t>(255);
        return at;
    };
    L.status = take(256);
    L.rstd = take(T * 4);
    L.scores = take(T * E * 4);
    L.idx = take(T * k * 4);
    L.gates = take(T * k * 4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 4);
    L.row_token = take(T * k * 4);
    L.row_of = take(T * k * 4);
    L.masks = take(nblk * E * 8 * 4);
    L.hist = take(nblk * E * 4);
    L.blkoff = take(nblk * E * 4);
    L.seg_start = take((E + 1) * 4);
    L.seg_rows = take((E + 1) * 4);
    L.tile_start = take((E + 2) * 4);
    L.a = take(Rs * d * es);
    L.a_scales = take(fp8 ? Rs * (d / 128) * 4 : 0);
    L.h = take(Rs * de * es);
    L.h_scales = take(fp8 ? Rs * (de / 128) * 4 : 0);
    L.y = take(Rs * d * 2);
    L.total = off;
    return L;
}

template <class T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

int check_ws(const moe_shape *s, void *ws, size_t ws_bytes, Layout *L) {
    *L = layout(s);
    if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255)
        return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (ws_bytes < L->total)
        return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L->total);
    return MOE_OK;
}

#define CHECK_PTR(p)                                                                   \
    do {                                                                               \
        if (!(p)) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", #p);                  \
        if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
    } while (0)

#define RETURN_IF(call)            \
    do {                           \
        const int rc_ = (call);    \
        if (rc_ != MOE_OK) return rc_; \
    } while (0)

#define LAUNCH(call, what)                                   \
    do {                                                     \
        const cudaError_t e_ = (call);                       \
        if (e_ != cudaSuccess) return cuda_fail(e_, what);   \
    } while (0)

PermScratch perm_scratch(void *ws, const Layout &L, int tile_m = kTileM) {
    PermScratch p;
    p.tile_m = tile_m;
    p.masks = at<uint32_t>(ws, L.masks);
    p.hist = at<int32_t>(ws, L.hist);
    p.blkoff = at<int32_t>(ws, L.blkoff);
    p.seg_start = at<int32_t>(ws, L.seg_start);
    p.seg_rows = at<int32_t>(ws, L.seg_rows);
    p.tile_start = at<int32_t>(ws, L.tile_start);
    return p;
}

// Rows per grouped-GEMM tile.  With fp32 scales every 128-wide K block makes
// a round trip through the epilogue; a 64-row tile carries two K blocks per
// round trip (M=64 accumulators fill half of each TMEM lane quadrant), so a
// segment of r rows costs ceil(r/64) * K/256 round trips against
// ceil(r/128) * K/128 with 128-row tiles.  That wins for batches of at most
// 64 tokens, whose segments have a few rows each.  At 4096 tokens (~128 rows
// per expert) 64-row tiles were measured slower (gate/up GEMM 2.68 ms against
// 2.13): they make fewer round trips but load each weight tile once per 64
// rows instead of per 128.
int choose_tile_m(const moe_shape *s) {
    return (s->precision == MOE_FP8_BLOCK && s->T <= 64) ? 64 : 128;
}

int grouped(const moe_shape *s, const void *a, const float *a_scales, const void *w13,
            const float *w13_scales, const void *w2, const float *w2_scales, uint16_t *y,
            void *ws, const Layout &L, cudaStream_t st, int *launches, int tile_m) {
    const bool fp8 = is_fp8(s);
    const PermScratch ps = perm_scratch(ws, L, tile_m);
    const int Rs = s->T * (s->top_k + s->n_shared);
    GemmArgs g{};
    g.fp8 = fp8;
    g.rows_total = Rs;
    g.n_slots = s->n_experts + s->n_shared;
    g.n_segments = s->n_experts + s->n_shared;
    g.E = s->n_experts;
    g.seg_start = ps.seg_start;
    g.seg_rows = ps.seg_rows;
    g.tile_start = ps.tile_start;
    g.status = at<int>(ws, L.status);
    g.inject_fault = inject_gemm_fault() ? 1 : 0;
    g.ue8m0 = is_ue8m0(s);
    g.tile_m = tile_m;
    g.b_rowmajor = s->weight_layout == MOE_LAYOUT_ROWMAJOR;
    // gate/up GEMM + SwiGLU
    g.gate_up = true;
    g.a = a;
    g.a_scales = a_scales;
    g.b = w13;
    g.b_scales = w13_scales;
    g.out = at<uint8_t>(ws, L.h);
    g.out_scales = fp8 ? at<float>(ws, L.h_scales) : nullptr;
    g.K = s->d_model;
    g.N_out = s->d_expert;
    LAUNCH(launch_grouped_gemm(g, st, launches), "grouped gate/up GEMM");
    // down GEMM
    g.inject_fault = 0;
    g.gate_up = false;
    g.a = at<uint8_t>(ws, L.h);
    g.a_scales = fp8 ? at<float>(ws, L.h_scales) : nullptr;
    g.b = w2;
    g.b_scales = w2_scales;
    g.out = y;
    g.out_scales = nullptr;
    g.K = s->d_expert;
    g.N_out = s->d_model;
    LAUNCH(launch_grouped_gemm(g, st, launches), "grouped down GEMM");
    return MOE_OK;
}

int check_weights(const moe_shape *s, const void *w13, const float *w13s, const void *w2,
                  const float *w2s) {
    CHECK_PTR(w13);
    CHECK_PTR(w2);
    if (is_fp8(s)) {
        CHECK_PTR(w13s);
        CHECK_PTR(w2s);
    }
    return MOE_OK;
}

}  // namespace

// Hooks for entry points defined in other files of the library.
int record_error(int code, const char *msg) { return fail(code, "%s", msg); }
void record_launches(int n) { g_launches = n; }
int validate_shape(const moe_shape *s) { return check_shape(s); }
int validate_device() { return check_device(); }

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_shape *shape) {
    if (check_shape(shape) != MOE_OK) return 0;
    return layout(shape).total;
}

int moe_workspace_layout(const moe_shape *shape, moe_workspace_offsets *out) {
    RETURN_IF(check_shape(shape));
    if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
    const Layout L = layout(shape);
    out->status = L.status;
    out->scores = L.scores;
    out->topk_idx = L.idx;
    out->topk_w = L.gates;
    out->counts = L.counts;
    out->offsets = L.offsets;
    out->row_token = L.row_token;
    out->row_of = L.row_of;
    out->a = L.a;
    out->a_scales = L.a_scales;
    out->h = L.h;
    out->h_scales = L.h_scales;
    out->y = L.y;
    out->total = L.total;
    return MOE_OK;
}

int moe_route(const moe_shape *s, const uint16_t *x, const uint16_t *w_router, const float *bias,
              int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes, void *stream) {
    const CallRange nvtx_range("moe_route");
    RETURN_IF(check_shape(s));
    Layout L;
    RETURN_IF(check_ws(s, ws, ws_bytes, &L));
    if (s->T == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(x);
    CHECK_PTR(w_router);
    CHECK_PTR(bias);
    CHECK_PTR(topk_idx);
    CHECK_PTR(topk_w);
    RETURN_IF(check_device());
    int n = 0;
    LAUNCH(launch_router(x, w_router, bias, s->T, s->d_model, s->n_experts, s->top_k,
                         s->routed_scale, at<float>(ws, L.scores), topk_idx, topk_w,
                         static_cast<cudaStream_t>(stream), &n),
           "router");
    mark_launch(static_cast<cudaStream_t>(stream), n);
    g_launches = n;
    return MOE_OK;
}

int moe_permute(const moe_shape *s, const int32_t *topk_idx, int32_t *counts, int32_t *offsets,
                int32_t *row_token, int32_t *row_of, void *ws, size_t ws_bytes, void *stream) {
    const CallRange nvtx_range("moe_permute");
    RETURN_IF(check_shape(s));
    Layout L;
    RETURN_IF(check_ws(s, ws, ws_bytes, &L));
    CHECK_PTR(counts);
    CHECK_PTR(offsets);
    if (s->T == 0) {
        // empty input: zero counts and offsets, nothing else to write
        LAUNCH(cudaMemsetAsync(counts, 0, sizeof(int32_t) * s->n_experts,
                               static_cast<cudaStream_t>(stream)), "memset");
        LAUNCH(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (s->n_experts + 1),
                               static_cast<cudaStream_t>(stream)), "memset");
        g_launches = 0;
        return MOE_OK;
    }
    CHECK_PTR(topk_idx);
    CHECK_PTR(row_token);
    CHECK_PTR(row_of);
    RETURN_IF(check_device());
    int n = 0;
    LAUNCH(launch_permute(topk_idx, s->T, s->top_k, s->n_experts, s->n_shared,
                          perm_scratch(ws, L), counts, offsets, row_token, row_of,
                          at<int>(ws, L.status), static_cast<cudaStream_t>(stream), &n),
           "permute");
    mark_launch(static_cast<cudaStream_t>(stream), n);
    g_launches = n;
    return MOE_OK;
}

static int block_quant_entry(const uint16_t *in, int rows, int cols, int ld, int block_rows,
                      int out_layout, uint8_t *q, float *scales, void *stream, bool ue8m0) {
    const CallRange nvtx_range("fp8_block_quant");
    if (rows < 0 || cols <= 0 || cols % 128 || ld < cols || ld % 8)
        return fail(MOE_ERR_INVALID_ARG, "need rows >= 0, cols a positive multiple of 128, "
                                         "ld >= cols, ld % 8 == 0");
    if (block_rows != 1 && block_rows != 128)
        return fail(MOE_ERR_INVALID_ARG, "block_rows must be 1 or 128");
    if (out_layout != MOE_LAYOUT_ROWMAJOR && out_layout != MOE_LAYOUT_TILED)
        return fail(MOE_ERR_INVALID_ARG, "unknown out_layout %d", out_layout);
    if (out_layout == MOE_LAYOUT_TILED && (block_rows != 128 || rows % 128))
        return fail(MOE_ERR_INVALID_ARG, "tiled output needs block_rows 128 and rows % 128 == 0");
    if (rows == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(in);
    CHECK_PTR(q);
    CHECK_PTR(scales);
    RETURN_IF(check_device());
    int n = 0;
    LAUNCH(launch_block_quant(in, rows, cols, ld, block_rows, out_layout == MOE_LAYOUT_TILED, q,
                              scales, static_cast<cudaStream_t>(stream), &n, ue8m0),
           "fp8_block_quant");
    mark_launch(static_cast<cudaStream_t>(stream), n);
    g_launches = n;
    return MOE_OK;
}

int fp8_block_quant(const uint16_t *in, int rows, int cols, int ld, int block_rows,
                    int out_layout, uint8_t *q, float *scales, void *stream) {
    return block_quant_entry(in, rows, cols, ld, block_rows, out_layout, q, scales, stream, false);
}

int fp8_block_quant_ue8m0(const uint16_t *in, int rows, int cols, int ld, int block_rows,
                          int out_layout, uint8_t *q, float *scales, void *stream) {
    return block_quant_entry(in, rows, cols, ld, block_rows, out_layout, q, scales, stream, true);
}

int moe_pack_tiles(const void *src, int rows, int row_bytes, void *dst, void *stream) {
    const CallRange nvtx_range("moe_pack_tiles");
    if (rows < 0 || row_bytes <= 0 || rows % 128 || row_bytes % 128)
        return fail(MOE_ERR_INVALID_ARG, "rows and row_bytes must be multiples of 128");
    if (rows == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(src);
    CHECK_PTR(dst);
    RETURN_IF(check_device());
    int n = 0;
    LAUNCH(launch_pack_tiles(src, rows, row_bytes, dst, static_cast<cudaStream_t>(stream), &n),
           "moe_pack_tiles");
    mark_launch(static_cast<cudaStream_t>(stream), n);
    g_launches = n;
    return MOE_OK;
}

int moe_grouped_swiglu(const moe_shape *s, const void *a, const float *a_scales,
                       const int32_t *offsets, const void *w13, const float *w13_scales,
                       const void *w2, const float *w2_scales, uint16_t *y, void *ws,
                       size_t ws_bytes, void *stream) {
    const CallRange nvtx_range("moe_grouped_swiglu");
    RETURN_IF(check_shape(s));
    Layout L;
    RETURN_IF(check_ws(s, ws, ws_bytes, &L));
    if (s->T == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(a);
    if (is_fp8(s)) CHECK_PTR(a_scales);
    CHECK_PTR(offsets);
    CHECK_PTR(y);
    RETURN_IF(check_weights(s, w13, w13_scales, w2, w2_scales));
    RETURN_IF(check_device());
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    int n = 0;
    const int tile_m = choose_tile_m(s);
    LAUNCH(launch_tile_table(offsets, s->n_experts, s->T, s->top_k, s->n_shared,
                             perm_scratch(ws, L, tile_m), at<int>(ws, L.status), st, &n),
           "tile table");
    RETURN_IF(grouped(s, a, a_scales, w13, w13_scales, w2, w2_scales, y, ws, L, st, &n, tile_m));
    mark_launch(st, n);
    g_launches = n;
    return MOE_OK;
}

int moe_quant_scatter(const moe_shape *s, const uint16_t *x, const int32_t *row_of, void *a,
                      float *a_scales, void *stream) {
    const CallRange nvtx_range("moe_quant_scatter");
    RETURN_IF(check_shape(s));
    if (s->T == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(x);
    CHECK_PTR(row_of);
    CHECK_PTR(a);
    const bool fp8 = is_fp8(s);
    if (fp8) CHECK_PTR(a_scales);
    RETURN_IF(check_device());
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    int n = 0;
    if (fp8)
        LAUNCH(launch_quant_scatter(x, s->T, s->d_model, s->top_k, s->n_shared, row_of,
                                    static_cast<uint8_t *>(a), a_scales, st, &n, PreNorm{},
                                    is_ue8m0(s)),
               "quant_scatter");
    else
        LAUNCH(launch_scatter_bf16(x, s->T, s->d_model, s->top_k, s->n_shared, row_of,
                                   static_cast<uint16_t *>(a), st, &n, PreNorm{}),
               "scatter");
    mark_launch(st, n);
    g_launches = n;
    return MOE_OK;
}

int moe_ep_dispatch(const moe_shape *s, const void *a, const float *a_scales, int a_rows,
                    int n_blocks, const moe_ep_block *blocks, int world, void *const *recv_a,
                    float *const *recv_scales, const int *recv_capacity, void *stream) {
    const CallRange nvtx_range("moe_ep_dispatch");
    RETURN_IF(check_shape(s));
    if (world < 1 || world > MOE_EP_MAX_RANKS)
        return fail(MOE_ERR_INVALID_ARG, "world must be in 1..%d", MOE_EP_MAX_RANKS);
    if (n_blocks < 0 || n_blocks > MOE_EP_MAX_RANKS)
        return fail(MOE_ERR_INVALID_ARG, "n_blocks must be in 0..%d", MOE_EP_MAX_RANKS);
    if (a_rows < 0) return fail(MOE_ERR_INVALID_ARG, "a_rows < 0");
    if (n_blocks > 0 && (!blocks || !recv_a || !recv_capacity))
        return fail(MOE_ERR_INVALID_ARG, "blocks, recv_a and recv_capacity must not be NULL");
    const bool fp8 = is_fp8(s);
    EpDispatchArgs g{};
    g.n_blocks = n_blocks;
    g.row_bytes = s->d_model * (fp8 ? 1 : 2);
    g.n_scales = fp8 ? s->d_model / 128 : 0;
    int total = 0;
    for (int b = 0; b < n_blocks; ++b) {
        const moe_ep_block &k = blocks[b];
        if (k.rows < 0 || k.src_row < 0 || static_cast<long long>(k.src_row) + k.rows > a_rows)
            return fail(MOE_ERR_INVALID_ARG, "block %d: source rows outside the buffer", b);
        if (k.dst < 0 || k.dst >= world)
            return fail(MOE_ERR_INVALID_ARG, "block %d: destination rank %d out of range", b, k.dst);
        if (k.dst_row < 0 || static_cast<long long>(k.dst_row) + k.rows > recv_capacity[k.dst])
            return fail(MOE_ERR_INVALID_ARG, "block %d: receive rows outside rank %d's buffer", b,
                        k.dst);
        if (k.rows > 0) {
            if (!recv_a[k.dst] || !aligned16(recv_a[k.dst]))
                return fail(MOE_ERR_INVALID_ARG, "recv_a[%d] is NULL or not 16-byte aligned", k.dst);
            if (fp8 && (!recv_scales || !recv_scales[k.dst] ||
                        (reinterpret_cast<uintptr_t>(recv_scales[k.dst]) & 3)))
                return fail(MOE_ERR_INVALID_ARG, "recv_scales[%d] is NULL or misaligned", k.dst);
        }
        g.src_row[b] = k.src_row;
        g.dst[b] = k.dst;
        g.dst_row[b] = k.dst_row;
        g.prefix[b] = total;
        total += k.rows;
    }
    g.prefix[n_blocks] = total;
    for (int r = 0; r < world; ++r) {
        g.dst_a[r] = recv_a ? static_cast<uint8_t *>(recv_a[r]) : nullptr;
        g.dst_s[r] = (fp8 && recv_scales) ? recv_scales[r] : nullptr;
    }
    if (total == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(a);
    if (fp8) CHECK_PTR(a_scales);
    RETURN_IF(check_device());
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    int n = 0;
    LAUNCH(launch_ep_dispatch(a, fp8 ? a_scales : nullptr, g, st, &n), "ep dispatch");
    mark_launch(st, n);
    g_launches = n;
    return MOE_OK;
}

int moe_combine(const moe_shape *s, const uint16_t *y, const int32_t *row_of,
                const float *topk_w, uint16_t *out, void *stream) {
    const CallRange nvtx_range("moe_combine");
    RETURN_IF(check_shape(s));
    if (s->T == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(y);
    CHECK_PTR(row_of);
    CHECK_PTR(topk_w);
    CHECK_PTR(out);
    RETURN_IF(check_device());
    int n = 0;
    LAUNCH(launch_combine(y, row_of, topk_w, s->T, s->d_model, s->top_k, s->n_shared, out,
                          static_cast<cudaStream_t>(stream), &n),
           "combine");
    mark_launch(static_cast<cudaStream_t>(stream), n);
    g_launches = n;
    return MOE_OK;
}

}  // extern "C"

namespace moe {
namespace {

// The whole layer.  x is the FFN input, or with gamma set the residual stream
// h, normalised on the fly (pre-norm) and added back in the combine.
int forward_impl(const moe_shape *s, const uint16_t *x, const uint16_t *gamma, float eps,
                 const uint16_t *w_router, const float *bias, const void *w13,
                 const float *w13_scales, const void *w2, const float *w2_scales, uint16_t *out,
                 int32_t *topk_idx_out, void *ws, size_t ws_bytes, void *stream) {
    const CallRange nvtx_range(gamma ? "moe_forward_prenorm" : "moe_forward");
    RETURN_IF(check_shape(s));
    Layout L;
    RETURN_IF(check_ws(s, ws, ws_bytes, &L));
    if (s->T == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(x);
    CHECK_PTR(w_router);
    CHECK_PTR(bias);
    CHECK_PTR(out);
    if (topk_idx_out && !aligned16(topk_idx_out))
        return fail(MOE_ERR_INVALID_ARG, "topk_idx_out is not 16-byte aligned");
    if (gamma && !(eps >= 0.0f)) return fail(MOE_ERR_INVALID_ARG, "eps must be >= 0");
    RETURN_IF(check_weights(s, w13, w13_scales, w2, w2_scales));
    RETURN_IF(check_device());
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool fp8 = is_fp8(s);
    int32_t *idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
    float *gates = at<float>(ws, L.gates);
    int32_t *row_of = at<int32_t>(ws, L.row_of);
    int n = 0;
    PreNorm pn{};
    if (gamma) {
        float *rstd = at<float>(ws, L.rstd);
        LAUNCH(launch_rstd(x, s->T, s->d_model, eps, rstd, st, &n), "pre-norm statistics");
        pn.rstd = rstd;
        pn.gamma = gamma;
    }
    LAUNCH(launch_router(x, w_router, bias, s->T, s->d_model, s->n_experts, s->top_k,
                         s->routed_scale, at<float>(ws, L.scores), idx, gates, st, &n, pn),
           "router");
    const int tile_m = choose_tile_m(s);
    LAUNCH(launch_permute(idx, s->T, s->top_k, s->n_experts, s->n_shared, perm_scratch(ws, L, tile_m),
                          at<int32_t>(ws, L.counts), at<int32_t>(ws, L.offsets),
                          at<int32_t>(ws, L.row_token), row_of, at<int>(ws, L.status), st, &n),
           "permute");
    if (fp8)
        LAUNCH(launch_quant_scatter(x, s->T, s->d_model, s->top_k, s->n_shared, row_of,
                                    at<uint8_t>(ws, L.a), at<float>(ws, L.a_scales), st, &n, pn,
                                    is_ue8m0(s)),
               "quant_scatter");
    else
        LAUNCH(launch_scatter_bf16(x, s->T, s->d_model, s->top_k, s->n_shared, row_of,
                                   at<uint16_t>(ws, L.a), st, &n, pn),
               "scatter");
    uint16_t *y = at<uint16_t>(ws, L.y);
    RETURN_IF(grouped(s, at<uint8_t>(ws, L.a), fp8 ? at<float>(ws, L.a_scales) : nullptr, w13,
                      w13_scales, w2, w2_scales, y, ws, L, st, &n, tile_m));
    LAUNCH(launch_combine(y, row_of, gates, s->T, s->d_model, s->top_k, s->n_shared, out, st, &n,
                          gamma ? x : nullptr),
           "combine");
    mark_launch(st, n);
    g_launches = n;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" {

int moe_forward(const moe_shape *s, const uint16_t *x, const uint16_t *w_router,
                const float *bias, const void *w13, const float *w13_scales, const void *w2,
                const float *w2_scales, uint16_t *out, int32_t *topk_idx_out, void *ws,
                size_t ws_bytes, void *stream) {
    return forward_impl(s, x, nullptr, 0.0f, w_router, bias, w13, w13_scales, w2, w2_scales, out,
                        topk_idx_out, ws, ws_bytes, stream);
}

int moe_forward_prenorm(const moe_shape *s, const uint16_t *h, const uint16_t *gamma, float eps,
                        const uint16_t *w_router, const float *bias, const void *w13,
                        const float *w13_scales, const void *w2, const float *w2_scales,
                        uint16_t *out, int32_t *topk_idx_out, void *ws, size_t ws_bytes,
                        void *stream) {
    if (!gamma) return fail(MOE_ERR_INVALID_ARG, "gamma is NULL");
    if (!aligned16(gamma)) return fail(MOE_ERR_INVALID_ARG, "gamma is not 16-byte aligned");
    return forward_impl(s, h, gamma, eps, w_router, bias, w13, w13_scales, w2, w2_scales, out,
                        topk_idx_out, ws, ws_bytes, stream);
}

}  // extern "C"

// ------------------------------------------------------- dense FFN layer ---
namespace moe {
namespace {

int check_dense_shape(const moe_dense_shape *s) {
    if (!s) return fail(MOE_ERR_INVALID_ARG, "shape is NULL");
    if (s->T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0");
    if (s->d_model <= 0 || s->d_model % 256)
        return fail(MOE_ERR_INVALID_ARG, "d_model must be a positive multiple of 256");
    if (s->d_ff <= 0 || s->d_ff % 128)
        return fail(MOE_ERR_INVALID_ARG, "d_ff must be a positive multiple of 128");
    if (s->precision != MOE_BF16 && s->precision != MOE_FP8_BLOCK &&
        s->precision != MOE_FP8_UE8M0)
        return fail(MOE_ERR_INVALID_ARG, "unknown precision %d", s->precision);
    if (s->weight_layout != MOE_LAYOUT_ROWMAJOR && s->weight_layout != MOE_LAYOUT_TILED)
        return fail(MOE_ERR_INVALID_ARG, "unknown weight_layout %d", s->weight_layout);
    if (static_cast<long long>(s->T) * std::max(s->d_model, s->d_ff) > (1LL << 40) ||
        s->T > (1 << 30))
        return fail(MOE_ERR_INVALID_ARG, "T too large");
    return MOE_OK;
}

// Split K of the dense down GEMM.  Its output has only ceil(T/128) x
// d_model/256 tiles (28 for a batch of up to 128 tokens at d_model 7168), too
// few to keep the SMs streaming weights, so small batches split K into up to
// kDenseMaxSplit ranges, whose binary32 partial sums a reduce kernel adds in
// order.  The workspace reserves the partial sums for batches of at most
// kDenseSplitRows tokens; the split itself is chosen per launch from the
// device's SM count.
constexpr int kDenseMaxSplit = kMaxSplitK;
constexpr int kDenseSplitRows = 256;

struct DenseLayout {
    size_t status, rstd, a, a_scales, h, h_scales, partial, total;
};

DenseLayout dense_layout(const moe_dense_shape *s) {
    const size_t T = s->T, d = s->d_model, f = s->d_ff;
    const bool fp8 = s->precision != MOE_BF16;
    const size_t es = fp8 ? 1 : 2;
    const bool split = s->T <= kDenseSplitRows && s->precision != MOE_FP8_UE8M0;
    DenseLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~static_cast<size_t>(255);
        return at;
    };
    L.status = take(256);
    L.rstd = take(T * 4);
    L.a = take(T * d * es);
    L.a_scales = take(fp8 ? T * (d / 128) * 4 : 0);
    L.h = take(T * f * es);
    L.h_scales = take(fp8 ? T * (f / 128) * 4 : 0);
    L.partial = take(split ? kDenseMaxSplit * T * d * 4 : 0);
    L.total = off;
    return L;
}

// Workspace of moe_ep_grouped_swiglu: status word, the checked segment table
// (start, rows, tile prefix, slot, source, return row), H and its scales.
struct EpLayout {
    size_t status, table, ret_y, h, h_scales, total;
};

EpLayout ep_layout(const moe_shape *s, int rows, int n_seg) {
    const bool fp8 = is_fp8(s);
    const size_t de = s->d_expert, R = rows;
    EpLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~static_cast<size_t>(255);
        return at;
    };
    L.status = take(256);
    L.table = take(6 * (static_cast<size_t>(n_seg) + 1) * 4);
    L.ret_y = take(MOE_EP_MAX_RANKS * sizeof(void *));
    L.h = take(R * de * (fp8 ? 1 : 2));
    L.h_scales = take(fp8 ? R * (de / 128) * 4 : 0);
    L.total = off;
    return L;
}

int dense_ksplit(const moe_dense_shape *s) {
    if (s->T > kDenseSplitRows || s->precision == MOE_FP8_UE8M0) return 1;
    const int tiles = gemm_output_tiles(s->T, s->d_model);
    const int kb = s->precision == MOE_BF16 ? s->d_ff / 64 : s->d_ff / 128;
    int ks = num_sms() / std::max(tiles, 1);
    ks = std::min(ks, kDenseMaxSplit);
    ks = std::min(ks, kb / 2);  // at least two K blocks per range
    return std::max(ks, 1);
}

int dense_impl(const moe_dense_shape *s, const uint16_t *x, const uint16_t *gamma, float eps,
               const void *w13, const float *w13_scales, const void *w2, const float *w2_scales,
               uint16_t *out, void *ws, size_t ws_bytes, void *stream) {
    const CallRange nvtx_range(gamma ? "moe_dense_ffn_prenorm" : "moe_dense_ffn");
    RETURN_IF(check_dense_shape(s));
    const DenseLayout L = dense_layout(s);
    if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255)
        return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (ws_bytes < L.total)
        return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
    if (s->T == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(x);
    CHECK_PTR(out);
    CHECK_PTR(w13);
    CHECK_PTR(w2);
    const bool fp8 = s->precision != MOE_BF16;
    const bool ue = s->precision == MOE_FP8_UE8M0;
    if (fp8) {
        CHECK_PTR(w13_scales);
        CHECK_PTR(w2_scales);
    }
    if (gamma && !(eps >= 0.0f)) return fail(MOE_ERR_INVALID_ARG, "eps must be >= 0");
    RETURN_IF(check_device());
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int T = s->T, d = s->d_model;
    int n = 0;
    PreNorm pn{};
    if (gamma) {
        float *rstd = at<float>(ws, L.rstd);
        LAUNCH(launch_rstd(x, T, d, eps, rstd, st, &n), "pre-norm statistics");
        pn.rstd = rstd;
        pn.gamma = gamma;
    }
    // A: x quantised 1x128 (fp8), the normalised copy (bf16 pre-norm), or x itself
    const void *a = x;
    if (fp8)
        LAUNCH(launch_quant_scatter(x, T, d, 0, 1, nullptr, at<uint8_t>(ws, L.a),
                                    at<float>(ws, L.a_scales), st, &n, pn, ue),
               "quantise x");
    else if (gamma)
        LAUNCH(launch_scatter_bf16(x, T, d, 0, 1, nullptr, at<uint16_t>(ws, L.a), st, &n, pn),
               "pre-norm x");
    if (fp8 || gamma) a = at<uint8_t>(ws, L.a);
    const int ks = dense_ksplit(s);
    GemmArgs g{};
    g.fp8 = fp8;
    g.rows_total = T;
    g.n_slots = 1;
    g.n_segments = 1;
    g.E = 0;
    g.seg_start = g.seg_rows = g.tile_start = nullptr;  // one segment of all T rows
    g.status = at<int>(ws, L.status);
    g.ue8m0 = ue;
    g.b_rowmajor = s->weight_layout == MOE_LAYOUT_ROWMAJOR;
    // one segment of T rows: 64-row tiles only where they save round trips
    g.tile_m = (s->precision == MOE_FP8_BLOCK && T <= 64) ? 64 : 128;
    g.gate_up = true;
    g.a = a;
    g.a_scales = fp8 ? at<float>(ws, L.a_scales) : nullptr;
    g.b = w13;
    g.b_scales = w13_scales;
    g.out = at<uint8_t>(ws, L.h);
    g.out_scales = fp8 ? at<float>(ws, L.h_scales) : nullptr;
    g.K = d;
    g.N_out = s->d_ff;
    LAUNCH(launch_grouped_gemm(g, st, &n), "dense gate/up GEMM");
    g.gate_up = false;
    g.a = at<uint8_t>(ws, L.h);
    g.a_scales = fp8 ? at<float>(ws, L.h_scales) : nullptr;
    g.b = w2;
    g.b_scales = w2_scales;
    g.out = out;
    g.out_scales = nullptr;
    g.K = s->d_ff;
    g.N_out = d;
    g.ksplit = ks;
    g.partial = ks > 1 ? at<float>(ws, L.partial) : nullptr;
    g.residual = gamma ? x : nullptr;
    LAUNCH(launch_grouped_gemm(g, st, &n), "dense down GEMM");
    if (ks > 1)
        LAUNCH(launch_splitk_reduce(at<float>(ws, L.partial), ks, T, d, gamma ? x : nullptr, out,
                                    st, &n),
               "split-K reduce");
    mark_launch(st, n);
    g_launches = n;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" {

size_t moe_dense_workspace_size(const moe_dense_shape *shape) {
    if (check_dense_shape(shape) != MOE_OK) return 0;
    return dense_layout(shape).total;
}

int moe_dense_ffn(const moe_dense_shape *s, const uint16_t *x, const void *w13,
                  const float *w13_scales, const void *w2, const float *w2_scales,
                  uint16_t *out, void *ws, size_t ws_bytes, void *stream) {
    return dense_impl(s, x, nullptr, 0.0f, w13, w13_scales, w2, w2_scales, out, ws, ws_bytes,
                      stream);
}

int moe_dense_ffn_prenorm(const moe_dense_shape *s, const uint16_t *h, const uint16_t *gamma,
                          float eps, const void *w13, const float *w13_scales, const void *w2,
                          const float *w2_scales, uint16_t *out, void *ws, size_t ws_bytes,
                          void *stream) {
    if (!gamma) return fail(MOE_ERR_INVALID_ARG, "gamma is NULL");
    return dense_impl(s, h, gamma, eps, w13, w13_scales, w2, w2_scales, out, ws, ws_bytes, stream);
}

size_t moe_ep_workspace_size(const moe_shape *s, int rows, int n_segments) {
    if (check_shape(s) != MOE_OK) return 0;
    if (rows < 0 || n_segments < 1 || n_segments > 1024) {
        fail(MOE_ERR_INVALID_ARG, "need rows >= 0 and 1 <= n_segments <= 1024");
        return 0;
    }
    return ep_layout(s, rows, n_segments).total;
}

int moe_ep_grouped_swiglu(const moe_shape *s, int rows, const void *a, const float *a_scales,
                          int n_segments, const int32_t *seg_start, const int32_t *seg_rows,
                          const int32_t *seg_slot, const int32_t *seg_src, const int32_t *seg_ret,
                          int n_slots, const void *w13, const float *w13_scales, const void *w2,
                          const float *w2_scales, int world, uint16_t *const *ret_y,
                          const int *ret_capacity, void *ws, size_t ws_bytes, void *stream) {
    const CallRange nvtx_range("moe_ep_grouped_swiglu");
    RETURN_IF(check_shape(s));
    if (rows < 0) return fail(MOE_ERR_INVALID_ARG, "rows < 0");
    if (n_segments < 1 || n_segments > 1024)
        return fail(MOE_ERR_INVALID_ARG, "n_segments must be in 1..1024");
    if (n_slots < 1 || n_slots > 1024) return fail(MOE_ERR_INVALID_ARG, "n_slots must be in 1..1024");
    if (world < 1 || world > MOE_EP_MAX_RANKS)
        return fail(MOE_ERR_INVALID_ARG, "world must be in 1..%d", MOE_EP_MAX_RANKS);
    const EpLayout L = ep_layout(s, rows, n_segments);
    if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255)
        return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (ws_bytes < L.total)
        return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
    if (rows == 0) return g_launches = 0, MOE_OK;
    CHECK_PTR(a);
    if (is_fp8(s)) CHECK_PTR(a_scales);
    CHECK_PTR(seg_start);
    CHECK_PTR(seg_rows);
    CHECK_PTR(seg_src);
    CHECK_PTR(seg_ret);
    if (seg_slot && !aligned16(seg_slot))
        return fail(MOE_ERR_INVALID_ARG, "seg_slot is not 16-byte aligned");
    if (!ret_y || !ret_capacity) return fail(MOE_ERR_INVALID_ARG, "ret_y and ret_capacity are NULL");
    for (int r = 0; r < world; ++r) {
        if (ret_capacity[r] < 0) return fail(MOE_ERR_INVALID_ARG, "ret_capacity[%d] < 0", r);
        // a source with no rows (capacity 0) may pass NULL; nothing returns to it
        if (ret_capacity[r] > 0 && (!ret_y[r] || !aligned16(ret_y[r])))
            return fail(MOE_ERR_INVALID_ARG, "ret_y[%d] is NULL or not 16-byte aligned", r);
    }
    RETURN_IF(check_weights(s, w13, w13_scales, w2, w2_scales));
    RETURN_IF(check_device());
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool fp8 = is_fp8(s);
    int n = 0;
    EpTableArgs t{};
    t.start = seg_start;
    t.rows = seg_rows;
    t.slot = seg_slot;
    t.src = seg_src;
    t.ret = seg_ret;
    t.n_seg = n_segments;
    t.rows_total = rows;
    t.n_slots = n_slots;
    t.world = world;
    t.tile_m = kTileM;
    for (int r = 0; r < world; ++r) {
        t.ret_capacity[r] = ret_capacity[r];
        t.ret_y[r] = ret_y[r];
    }
    int32_t *tab = at<int32_t>(ws, L.table);
    const size_t S = static_cast<size_t>(n_segments) + 1;
    int32_t *v_start = tab, *v_rows = tab + S, *v_tiles = tab + 2 * S, *v_slot = tab + 3 * S,
            *v_src = tab + 4 * S, *v_ret = tab + 5 * S;
    uint16_t **ret_dev = at<uint16_t *>(ws, L.ret_y);
    LAUNCH(launch_ep_table(t, v_start, v_rows, v_tiles, v_slot, v_src, v_ret, ret_dev,
                           at<int>(ws, L.status), st, &n),
           "ep segment table");
    GemmArgs g{};
    g.fp8 = fp8;
    g.rows_total = rows;
    g.n_slots = n_slots;
    g.n_segments = n_segments;
    g.E = n_segments;
    g.seg_start = v_start;
    g.seg_rows = v_rows;
    g.tile_start = v_tiles;
    g.seg_slot = v_slot;
    g.status = at<int>(ws, L.status);
    g.inject_fault = 0;
    g.ue8m0 = is_ue8m0(s);
    g.tile_m = kTileM;
    g.b_rowmajor = s->weight_layout == MOE_LAYOUT_ROWMAJOR;
    g.gate_up = true;
    g.a = a;
    g.a_scales = a_scales;
    g.b = w13;
    g.b_scales = w13_scales;
    g.out = at<uint8_t>(ws, L.h);
    g.out_scales = fp8 ? at<float>(ws, L.h_scales) : nullptr;
    g.K = s->d_model;
    g.N_out = s->d_expert;
    LAUNCH(launch_grouped_gemm(g, st, &n), "EP gate/up GEMM");
    // down GEMM: Y rows straight into the source ranks' buffers
    g.gate_up = false;
    g.a = at<uint8_t>(ws, L.h);
    g.a_scales = fp8 ? at<float>(ws, L.h_scales) : nullptr;
    g.b = w2;
    g.b_scales = w2_scales;
    g.out = ret_y[0];
    g.out_scales = nullptr;
    g.K = s->d_expert;
    g.N_out = s->d_model;
    g.seg_src = v_src;
    g.seg_ret = v_ret;
    g.ret_y_dev = ret_dev;
    LAUNCH(launch_grouped_gemm(g, st, &n), "EP down GEMM");
    mark_launch(st, n);
    g_launches = n;
    return MOE_OK;
}

int moe_check_status(void *ws, void *stream) {
    if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    int h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "moe_check_status");
    if (h != MOE_OK) {
        const int zero = 0;
        e = cudaMemcpyAsync(ws, &zero, sizeof(int), cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "moe_check_status reset");
        return fail(h, "device status %d", h);
    }
    return MOE_OK;
}

const char *moe_last_error(void) { return g_err.c_str(); }

int moe_last_launch_count(void) { return g_launches; }

const char *moe_last_launch_name(int i) {
    return (i >= 0 && i < g_launches && i < kMaxNamed) ? g_names[i] : nullptr;
}

int moe_set_kernel_events(void **events, int n_events) {
    if (events && n_events <= 0) return fail(MOE_ERR_INVALID_ARG, "n_events must be positive");
    g_events = reinterpret_cast<cudaEvent_t *>(events);
    g_n_events = events ? n_events : 0;
    return MOE_OK;
}

}  // extern "C"
