"""ctypes binding of libmoe_fwd.so (include/moe_fwd.h): argument marshalling
only.  Every computation of the layer runs in the library's CUDA kernels;
torch supplies device memory and the current stream.  There is no fallback:
if the library is missing or fails to load, every call raises."""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_fwd.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_TIMEOUT = -5
MOE_ERR_DEVICE_INDEX = -6
MOE_BF16 = 0
MOE_FP8_BLOCK = 1
MOE_FP8_UE8M0 = 2
MOE_LAYOUT_ROWMAJOR = 0
MOE_LAYOUT_TILED = 1

# every symbol include/moe_fwd.h declares
EXPORTS = ("moe_workspace_size", "moe_route", "moe_permute", "fp8_block_quant",
           "moe_grouped_swiglu", "moe_combine", "moe_forward", "moe_check_status",
           "moe_last_error", "moe_last_launch_count", "moe_set_kernel_events",
           "moe_route_noalloc", "moe_pack_tiles", "moe_forward_prenorm", "moe_last_launch_name",
           "fp8_block_quant_ue8m0", "moe_dense_workspace_size", "moe_dense_ffn",
           "moe_dense_ffn_prenorm", "moe_workspace_layout", "moe_quant_scatter",
           "moe_ep_dispatch", "moe_ep_workspace_size", "moe_ep_grouped_swiglu")

MOE_EP_MAX_RANKS = 64

# fixed score scratch of moe_route_noalloc, in floats (include/moe_fwd.h)
MOE_ROUTE_NOALLOC_MAX_SCORES = 1 << 20


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("d_model", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("d_expert", ctypes.c_int), ("n_shared", ctypes.c_int),
                ("routed_scale", ctypes.c_float), ("precision", ctypes.c_int),
                ("weight_layout", ctypes.c_int)]


class MoeDenseShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("d_model", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("precision", ctypes.c_int), ("weight_layout", ctypes.c_int)]


class MoeEpBlock(ctypes.Structure):
    _fields_ = [("src_row", ctypes.c_int), ("rows", ctypes.c_int), ("dst", ctypes.c_int),
                ("dst_row", ctypes.c_int)]


class MoeWorkspaceOffsets(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "status", "scores", "topk_idx", "topk_w", "counts", "offsets", "row_token", "row_of",
        "a", "a_scales", "h", "h_scales", "y", "total")]


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"moe_fwd error {code}: {msg}")
        self.code = code


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (built in-tree by build.py)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} not built: run sparse_moe_transformer_fwd_b200/build.py "
                              "(or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, ci, cf = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
        sp = ctypes.POINTER(MoeShape)
        L.moe_workspace_size.argtypes = [sp]
        L.moe_workspace_size.restype = sz
        L.moe_workspace_layout.argtypes = [sp, ctypes.POINTER(MoeWorkspaceOffsets)]
        L.moe_quant_scatter.argtypes = [sp, vp, vp, vp, vp, vp]
        pp = ctypes.POINTER(ctypes.c_void_p)
        ip = ctypes.POINTER(ctypes.c_int)
        L.moe_ep_dispatch.argtypes = [sp, vp, vp, ci, ci, ctypes.POINTER(MoeEpBlock), ci, pp, pp,
                                      ip, vp]
        L.moe_ep_workspace_size.argtypes = [sp, ci, ci]
        L.moe_ep_workspace_size.restype = sz
        L.moe_ep_grouped_swiglu.argtypes = [sp, ci, vp, vp, ci, vp, vp, vp, vp, vp, ci, vp, vp, vp,
                                            vp, ci, pp, ip, vp, sz, vp]
        L.moe_route.argtypes = [sp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_permute.argtypes = [sp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_route_noalloc.argtypes = [sp, vp, vp, vp, vp, vp, vp]
        L.fp8_block_quant.argtypes = [vp, ci, ci, ci, ci, ci, vp, vp, vp]
        L.fp8_block_quant_ue8m0.argtypes = [vp, ci, ci, ci, ci, ci, vp, vp, vp]
        L.moe_pack_tiles.argtypes = [vp, ci, ci, vp, vp]
        L.moe_grouped_swiglu.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_combine.argtypes = [sp, vp, vp, vp, vp, vp]
        L.moe_forward.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_forward_prenorm.argtypes = [sp, vp, vp, cf, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        dp = ctypes.POINTER(MoeDenseShape)
        L.moe_dense_workspace_size.argtypes = [dp]
        L.moe_dense_workspace_size.restype = sz
        L.moe_dense_ffn.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_dense_ffn_prenorm.argtypes = [dp, vp, vp, cf, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_check_status.argtypes = [vp, vp]
        L.moe_last_error.argtypes = []
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_last_launch_count.argtypes = []
        L.moe_last_launch_name.argtypes = [ci]
        L.moe_last_launch_name.restype = ctypes.c_char_p
        L.moe_set_kernel_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ci]
        for name in ("moe_route", "moe_route_noalloc", "moe_permute", "fp8_block_quant",
                     "fp8_block_quant_ue8m0", "moe_grouped_swiglu",
                     "moe_combine", "moe_forward", "moe_check_status", "moe_last_launch_count",
                     "moe_set_kernel_events", "moe_pack_tiles", "moe_forward_prenorm",
                     "moe_dense_ffn", "moe_dense_ffn_prenorm", "moe_workspace_layout",
                     "moe_quant_scatter", "moe_ep_dispatch", "moe_ep_grouped_swiglu"):
            getattr(L, name).restype = ci
        _LIB = L
    return _LIB


def _check(rc: int) -> None:
    if rc != MOE_OK:
        raise MoeError(rc, lib().moe_last_error().decode())


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _layout(weight_layout) -> int:
    return {"rowmajor": MOE_LAYOUT_ROWMAJOR, "tiled": MOE_LAYOUT_TILED}[weight_layout] \
        if isinstance(weight_layout, str) else int(weight_layout)


def make_shape(T, d_model, n_experts, top_k, d_expert, n_shared=1, routed_scale=1.0,
               precision="fp8", weight_layout=MOE_LAYOUT_TILED) -> MoeShape:
    prec = {"bf16": MOE_BF16, "fp8": MOE_FP8_BLOCK, "fp8_ue8m0": MOE_FP8_UE8M0}[precision] \
        if isinstance(precision, str) \
        else int(precision)
    return MoeShape(int(T), int(d_model), int(n_experts), int(top_k), int(d_expert),
                    int(n_shared), float(routed_scale), prec, _layout(weight_layout))


def make_dense_shape(T, d_model, d_ff, precision="fp8",
                     weight_layout=MOE_LAYOUT_TILED) -> MoeDenseShape:
    prec = {"bf16": MOE_BF16, "fp8": MOE_FP8_BLOCK, "fp8_ue8m0": MOE_FP8_UE8M0}[precision] \
        if isinstance(precision, str) else int(precision)
    return MoeDenseShape(int(T), int(d_model), int(d_ff), prec, _layout(weight_layout))


def moe_workspace_layout(shape: MoeShape) -> dict:
    """Byte offsets of moe_forward's intermediate results in its workspace."""
    o = MoeWorkspaceOffsets()
    _check(lib().moe_workspace_layout(ctypes.byref(shape), ctypes.byref(o)))
    return {n: getattr(o, n) for n, _ in MoeWorkspaceOffsets._fields_}


_BF16 = torch.bfloat16
_FP8 = (torch.uint8, torch.float8_e4m3fn)


def moe_workspace_size(shape: MoeShape) -> int:
    n = lib().moe_workspace_size(ctypes.byref(shape))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, lib().moe_last_error().decode())
    return n


def alloc_workspace(shape: MoeShape, device="cuda") -> torch.Tensor:
    """A zero-filled workspace (zero status word) of moe_workspace_size bytes."""
    return torch.zeros(moe_workspace_size(shape), dtype=torch.uint8, device=device)


def moe_route(shape, x, w_router, bias, topk_idx, topk_w, ws, stream=None):
    _check(lib().moe_route(ctypes.byref(shape), _ptr(x, _BF16, "x"),
                           _ptr(w_router, _BF16, "w_router"), _ptr(bias, torch.float32, "bias"),
                           _ptr(topk_idx, torch.int32, "topk_idx"),
                           _ptr(topk_w, torch.float32, "topk_w"), _ptr(ws, torch.uint8, "ws"),
                           ws.numel(), _stream(stream)))


def moe_route_noalloc(shape, x, w_router, bias, topk_idx, topk_w, stream=None):
    """moe_route without a workspace: for callers that may not allocate device
    memory.  The [T, E] score scratch is a fixed array inside the library
    (T * E <= MOE_ROUTE_NOALLOC_MAX_SCORES); calls that overlap on the GPU race."""
    _check(lib().moe_route_noalloc(ctypes.byref(shape), _ptr(x, _BF16, "x"),
                                   _ptr(w_router, _BF16, "w_router"),
                                   _ptr(bias, torch.float32, "bias"),
                                   _ptr(topk_idx, torch.int32, "topk_idx"),
                                   _ptr(topk_w, torch.float32, "topk_w"), _stream(stream)))


def moe_permute(shape, topk_idx, counts, offsets, row_token, row_of, ws, stream=None):
    i32 = torch.int32
    _check(lib().moe_permute(ctypes.byref(shape), _ptr(topk_idx, i32, "topk_idx"),
                             _ptr(counts, i32, "counts"), _ptr(offsets, i32, "offsets"),
                             _ptr(row_token, i32, "row_token"), _ptr(row_of, i32, "row_of"),
                             _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def fp8_block_quant(inp, block_rows, q, scales, rows=None, cols=None, ld=None,
                    layout=MOE_LAYOUT_ROWMAJOR, stream=None, ue8m0=False):
    """e4m3 block quantisation of a bf16 matrix (2-D, or a stack flattened to
    2-D); layout MOE_LAYOUT_TILED writes the codes in 128 x 128 tiles;
    ue8m0 selects power-of-two scales (fp8_block_quant_ue8m0)."""
    cols = inp.shape[-1] if cols is None else cols
    rows = inp.numel() // inp.shape[-1] if rows is None else rows
    ld = inp.shape[-1] if ld is None else ld
    fn = lib().fp8_block_quant_ue8m0 if ue8m0 else lib().fp8_block_quant
    _check(fn(_ptr(inp, _BF16, "in"), rows, cols, ld, block_rows, int(layout),
              _ptr(q, _FP8, "q"), _ptr(scales, torch.float32, "scales"), _stream(stream)))


def moe_pack_tiles(src, dst, stream=None):
    """Row-major -> 128 x 128-byte tiles (MOE_LAYOUT_TILED) of a matrix, or a
    stack of matrices flattened to rows x row_bytes; same shape and dtype."""
    if src.shape != dst.shape or src.dtype != dst.dtype:
        raise ValueError("src and dst must have the same shape and dtype")
    row_bytes = src.shape[-1] * src.element_size()
    rows = src.numel() // src.shape[-1]
    _check(lib().moe_pack_tiles(_ptr(src, name="src"), rows, row_bytes, _ptr(dst, name="dst"),
                                _stream(stream)))


def moe_grouped_swiglu(shape, a, a_scales, offsets, w13, w13_scales, w2, w2_scales, y, ws,
                       stream=None):
    fp8 = shape.precision in (MOE_FP8_BLOCK, MOE_FP8_UE8M0)
    wt = _FP8 if fp8 else _BF16
    _check(lib().moe_grouped_swiglu(
        ctypes.byref(shape), _ptr(a, wt, "a"), _ptr(a_scales, torch.float32, "a_scales"),
        _ptr(offsets, torch.int32, "offsets"), _ptr(w13, wt, "w13"),
        _ptr(w13_scales, torch.float32, "w13_scales"), _ptr(w2, wt, "w2"),
        _ptr(w2_scales, torch.float32, "w2_scales"), _ptr(y, _BF16, "y"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_combine(shape, y, row_of, topk_w, out, stream=None):
    _check(lib().moe_combine(ctypes.byref(shape), _ptr(y, _BF16, "y"),
                             _ptr(row_of, torch.int32, "row_of"),
                             _ptr(topk_w, torch.float32, "topk_w"), _ptr(out, _BF16, "out"),
                             _stream(stream)))


def moe_forward(shape, x, w_router, bias, w13, w13_scales, w2, w2_scales, out, ws,
                topk_idx_out=None, stream=None):
    fp8 = shape.precision in (MOE_FP8_BLOCK, MOE_FP8_UE8M0)
    wt = _FP8 if fp8 else _BF16
    _check(lib().moe_forward(
        ctypes.byref(shape), _ptr(x, _BF16, "x"), _ptr(w_router, _BF16, "w_router"),
        _ptr(bias, torch.float32, "bias"), _ptr(w13, wt, "w13"),
        _ptr(w13_scales, torch.float32, "w13_scales"), _ptr(w2, wt, "w2"),
        _ptr(w2_scales, torch.float32, "w2_scales"), _ptr(out, _BF16, "out"),
        _ptr(topk_idx_out, torch.int32, "topk_idx_out"), _ptr(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream)))


def moe_forward_prenorm(shape, h, gamma, eps, w_router, bias, w13, w13_scales, w2, w2_scales, out,
                        ws, topk_idx_out=None, stream=None):
    """out = h + MoE(bf16(RMSNorm(h) * gamma)); x is never materialised."""
    fp8 = shape.precision in (MOE_FP8_BLOCK, MOE_FP8_UE8M0)
    wt = _FP8 if fp8 else _BF16
    _check(lib().moe_forward_prenorm(
        ctypes.byref(shape), _ptr(h, _BF16, "h"), _ptr(gamma, _BF16, "gamma"), float(eps),
        _ptr(w_router, _BF16, "w_router"), _ptr(bias, torch.float32, "bias"), _ptr(w13, wt, "w13"),
        _ptr(w13_scales, torch.float32, "w13_scales"), _ptr(w2, wt, "w2"),
        _ptr(w2_scales, torch.float32, "w2_scales"), _ptr(out, _BF16, "out"),
        _ptr(topk_idx_out, torch.int32, "topk_idx_out"), _ptr(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream)))


def moe_dense_workspace_size(shape: MoeDenseShape) -> int:
    n = lib().moe_dense_workspace_size(ctypes.byref(shape))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, lib().moe_last_error().decode())
    return n


def alloc_dense_workspace(shape: MoeDenseShape, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of moe_dense_workspace_size bytes."""
    return torch.zeros(moe_dense_workspace_size(shape), dtype=torch.uint8, device=device)


def moe_dense_ffn(shape, x, w13, w13_scales, w2, w2_scales, out, ws, stream=None):
    """Dense gated FFN layer: out = (silu(x Wg^T) * (x Wu^T)) W2^T."""
    wt = _FP8 if shape.precision in (MOE_FP8_BLOCK, MOE_FP8_UE8M0) else _BF16
    _check(lib().moe_dense_ffn(
        ctypes.byref(shape), _ptr(x, _BF16, "x"), _ptr(w13, wt, "w13"),
        _ptr(w13_scales, torch.float32, "w13_scales"), _ptr(w2, wt, "w2"),
        _ptr(w2_scales, torch.float32, "w2_scales"), _ptr(out, _BF16, "out"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_dense_ffn_prenorm(shape, h, gamma, eps, w13, w13_scales, w2, w2_scales, out, ws,
                          stream=None):
    """out = h + FFN(bf16(RMSNorm(h) * gamma)), one final rounding."""
    wt = _FP8 if shape.precision in (MOE_FP8_BLOCK, MOE_FP8_UE8M0) else _BF16
    _check(lib().moe_dense_ffn_prenorm(
        ctypes.byref(shape), _ptr(h, _BF16, "h"), _ptr(gamma, _BF16, "gamma"), float(eps),
        _ptr(w13, wt, "w13"), _ptr(w13_scales, torch.float32, "w13_scales"), _ptr(w2, wt, "w2"),
        _ptr(w2_scales, torch.float32, "w2_scales"), _ptr(out, _BF16, "out"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_quant_scatter(shape, x, row_of, a, a_scales, stream=None):
    """x quantised 1x128 (or copied, bf16) into the permuted rows of `a`."""
    fp8 = shape.precision in (MOE_FP8_BLOCK, MOE_FP8_UE8M0)
    _check(lib().moe_quant_scatter(ctypes.byref(shape), _ptr(x, _BF16, "x"),
                                   _ptr(row_of, torch.int32, "row_of"),
                                   _ptr(a, _FP8 if fp8 else _BF16, "a"),
                                   _ptr(a_scales, torch.float32, "a_scales"), _stream(stream)))


def _ptr_array(tensors, dtype=None, name="tensor"):
    arr = (ctypes.c_void_p * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = _ptr(t, dtype, f"{name}[{i}]").value if t is not None else None
    return arr


def moe_ep_dispatch(shape, a, a_scales, blocks, recv_a, recv_scales=None, stream=None):
    """Copies blocks [(src_row, rows, dst, dst_row)] of the source's permuted
    rows `a` (and scales) into the owners' receive buffers recv_a[dst]."""
    fp8 = shape.precision in (MOE_FP8_BLOCK, MOE_FP8_UE8M0)
    world = len(recv_a)
    blk = (MoeEpBlock * max(1, len(blocks)))(*[MoeEpBlock(*map(int, b)) for b in blocks])
    cap = (ctypes.c_int * world)(*[int(t.shape[0]) for t in recv_a])
    ra = _ptr_array(recv_a, _FP8 if fp8 else _BF16, "recv_a")
    rs = _ptr_array(recv_scales, torch.float32, "recv_scales") if recv_scales is not None else None
    _check(lib().moe_ep_dispatch(ctypes.byref(shape), _ptr(a, _FP8 if fp8 else _BF16, "a"),
                                 _ptr(a_scales, torch.float32, "a_scales"), int(a.shape[0]),
                                 len(blocks), blk, world, ra, rs, cap, _stream(stream)))


def moe_ep_workspace_size(shape, rows: int, n_segments: int) -> int:
    n = lib().moe_ep_workspace_size(ctypes.byref(shape), int(rows), int(n_segments))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, lib().moe_last_error().decode())
    return n


def moe_ep_grouped_swiglu(shape, a, a_scales, seg_start, seg_rows, seg_slot, seg_src, seg_ret,
                          n_slots, w13, w13_scales, w2, w2_scales, ret_y, ws, stream=None):
    """Grouped gated MLP over the segments of `a`; row j of segment i is
    stored in ret_y[seg_src[i]] at row seg_ret[i] + (j - seg_start[i])."""
    fp8 = shape.precision in (MOE_FP8_BLOCK, MOE_FP8_UE8M0)
    wt = _FP8 if fp8 else _BF16
    world = len(ret_y)
    cap = (ctypes.c_int * world)(*[int(t.shape[0]) for t in ret_y])
    i32 = torch.int32
    _check(lib().moe_ep_grouped_swiglu(
        ctypes.byref(shape), int(a.shape[0]), _ptr(a, wt, "a"),
        _ptr(a_scales, torch.float32, "a_scales"), int(seg_start.numel()),
        _ptr(seg_start, i32, "seg_start"), _ptr(seg_rows, i32, "seg_rows"),
        _ptr(seg_slot, i32, "seg_slot"), _ptr(seg_src, i32, "seg_src"),
        _ptr(seg_ret, i32, "seg_ret"), int(n_slots), _ptr(w13, wt, "w13"),
        _ptr(w13_scales, torch.float32, "w13_scales"), _ptr(w2, wt, "w2"),
        _ptr(w2_scales, torch.float32, "w2_scales"), world, _ptr_array(ret_y, _BF16, "ret_y"),
        cap, _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_check_status(ws, stream=None) -> int:
    """Synchronises the stream; returns (and clears) the workspace status word."""
    return lib().moe_check_status(_ptr(ws, torch.uint8, "ws"), _stream(stream))


def moe_last_error() -> str:
    return lib().moe_last_error().decode()


def moe_last_launch_count() -> int:
    return lib().moe_last_launch_count()


def moe_last_launch_names() -> list:
    """Kernel names of the last call on this thread, in launch order."""
    L = lib()
    return [L.moe_last_launch_name(i).decode() for i in range(L.moe_last_launch_count())]


def moe_set_kernel_events(events) -> None:
    """Profiling hook: `events` is a list of torch.cuda.Event (created with
    enable_timing=True; None entries are skipped) or None to switch it off.
    Later calls on this thread record events[i] before their i-th kernel
    launch and events[launches] after the last."""
    if events is None:
        _check(lib().moe_set_kernel_events(None, 0))
        return
    for e in events:  # torch creates the CUDA event lazily, on its first record
        if e is not None and e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * len(events))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else None) for e in events])
    moe_set_kernel_events._keep = arr  # the library keeps the pointer
    _check(lib().moe_set_kernel_events(arr, len(events)))
