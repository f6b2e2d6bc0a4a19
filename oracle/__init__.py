"""Oracle for the DeepSeek-V3/R1 MoE FFN layer forward (CPU, plain, slow).

TEST INFRASTRUCTURE ONLY: the test-suite, the package smoke check and the
benchmark's CPU-baseline leg may use this package; the product path never
imports, loads or calls it.  It shares no code with the CUDA library.

What the layer computes, step by step, with the passage each step follows:

 1. Router logits l = x W_r^T (binary32, sequential fused multiply-add over
    d_model) and affinity s = sigmoid(l); selection score s + b where b is a
    per-expert bias used for routing only; top-k by (score desc, index asc);
    gates g_j = s_j / sum_selected(s) * routed_scale.
    ("DeepSeek v3 and R1 Model Architecture", section "Local Balanced Routing
    to Experts": token-to-expert affinity plus a routing-only bias term;
    "DeepSeek-R1" architecture card, "Every architecture field": 256 experts,
    8 active.)  C core: moe_oracle.c.
 2. Permutation: expert e's segment holds, in ascending token order, the
    tokens that selected e; segments are laid out in expert order; the shared
    expert's segment follows them and holds every token in order.  (Same page,
    "How is a token assigned to an expert"; card: 1 shared expert.)
 3. Blockwise e4m3 quantisation, 1x128 activation tiles and 128x128 weight
    blocks with binary32 scales ("DeepSeek-R1", aguasto.com, "Quantization":
    blockwise FP8).  C core.
 4. Gated experts (SwiGLU): H = silu(A W_gate^T) * (A W_up^T), Y = H W_down^T,
    d_expert 2048, d_model 7168 (card, "ffns.moe.gated", "ffns.moe.d_expert";
    "Architecture Overview" of the onlylabs page names SwiGLU).  In the FP8
    scheme every product is the real-valued product of the dequantised
    operands, evaluated in binary64 (numpy matmul); H is quantised 1x128 again
    before the down projection; Y is stored as bf16.  In the bf16 scheme H is
    rounded to bf16.
 5. Combine: out[t] = bf16( sum_j g[t,j] * Y[row(t,j)] + Y_shared[t] ) (the
    shared expert takes part in every token's output with weight 1: "DeepSeek v3
    and R1 Model Architecture", section "Structural change").

 6. Dense gated FFN of the first layers (card, "Every architecture field":
    layout 3 dense layers then 58 MoE layers; ffns.dense gated, d_ff 18432):
    one gated MLP as in step 4 over every token, out = bf16(Y).

The oracle mirrors every storage rounding of the layer (bf16 Y, bf16 or e4m3
H, bf16 out) and otherwise computes in binary64.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

__all__ = [
    "lib", "bf16_to_f32", "bf16_from_f32", "e4m3_decode_table", "e4m3_encode", "sigmoid",
    "router_logits", "route", "permute", "block_quant", "dequant", "expert_forward",
    "moe_layer", "exp_cw", "rmsnorm", "moe_layer_prenorm", "dense_ffn", "dense_ffn_prenorm",
    "h_code_ambiguity", "h_code_alternatives", "h_bf16_ambiguity", "h_bf16_alternatives",
]

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        f32p = ctypes.POINTER(ctypes.c_float)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i32p = ctypes.POINTER(ctypes.c_int32)
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_bf16_from_f32.argtypes = [ctypes.c_float]
        L.oracle_bf16_from_f32.restype = ctypes.c_uint16
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_float
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_exp_cw.argtypes = [ctypes.c_float]
        L.oracle_exp_cw.restype = ctypes.c_float
        L.oracle_sigmoid.argtypes = [ctypes.c_float]
        L.oracle_sigmoid.restype = ctypes.c_float
        L.oracle_block_quant.argtypes = [f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, u8p, f32p]
        L.oracle_block_quant.restype = None
        L.oracle_block_quant_ue8m0.argtypes = [f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, u8p,
                                               f32p]
        L.oracle_block_quant_ue8m0.restype = None
        L.oracle_router_logits.argtypes = [u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, f32p]
        L.oracle_router_logits.restype = None
        L.oracle_route.argtypes = [f32p, f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_float, i32p, f32p, f32p]
        L.oracle_route.restype = None
        L.oracle_bf16_from_f32_array.argtypes = [f32p, ctypes.c_size_t, u16p]
        L.oracle_e4m3_encode_array.argtypes = [f32p, ctypes.c_size_t, u8p]
        L.oracle_sigmoid_array.argtypes = [f32p, ctypes.c_size_t, f32p]
        L.oracle_rms_rstd.argtypes = [u16p, ctypes.c_int, ctypes.c_float]
        L.oracle_rms_rstd.restype = ctypes.c_float
        L.oracle_rmsnorm.argtypes = [u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_float, u16p, f32p]
        L.oracle_rmsnorm.restype = None
        _LIB = L
    return _LIB


def _p(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# ------------------------------------------------------------------ codecs --

def bf16_to_f32(h) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 (exact widening)."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def bf16_from_f32(f) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (C core)."""
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, dtype=np.uint16)
    lib().oracle_bf16_from_f32_array(_p(f, ctypes.c_float), f.size, _p(out, ctypes.c_uint16))
    return out


def e4m3_decode_table() -> np.ndarray:
    """binary64 value of each of the 256 e4m3 codes (NaN for S.1111.111)."""
    L = lib()
    return np.array([L.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(f) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(_p(f, ctypes.c_float), f.size, _p(out, ctypes.c_uint8))
    return out


def sigmoid(l) -> np.ndarray:
    l = np.ascontiguousarray(l, dtype=np.float32)
    out = np.empty(l.shape, dtype=np.float32)
    lib().oracle_sigmoid_array(_p(l, ctypes.c_float), l.size, _p(out, ctypes.c_float))
    return out


def exp_cw(y: float) -> float:
    return lib().oracle_exp_cw(float(y))


# ------------------------------------------------------------------ router --

def router_logits(x_bf16, w_router_bf16, workers: int = 1) -> np.ndarray:
    """[T, E] binary32 logits, sequential FMA over d_model (C core).
    workers > 1 splits the tokens into that many chunks, each one
    single-threaded call of the C core on its own thread (every logit is
    computed on its own, so the result does not depend on the split)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    w = np.ascontiguousarray(w_router_bf16, dtype=np.uint16)
    T, d = x.shape
    E = w.shape[0]
    out = np.empty((T, E), dtype=np.float32)

    def rows(lo, hi):
        lib().oracle_router_logits(_p(x[lo:hi], ctypes.c_uint16), _p(w, ctypes.c_uint16),
                                   hi - lo, d, E, _p(out[lo:hi], ctypes.c_float))

    workers = max(1, min(int(workers), T))
    if workers == 1:
        rows(0, T)
    else:
        import concurrent.futures as cf
        cuts = np.linspace(0, T, workers + 1).astype(int)
        with cf.ThreadPoolExecutor(workers) as ex:
            list(ex.map(lambda i: rows(cuts[i], cuts[i + 1]), range(workers)))
    return out


def route(logits, bias, k: int, routed_scale: float = 1.0):
    """-> (idx int32 [T,k] rank order, gates fp32 [T,k], scores fp32 [T,E])."""
    l = np.ascontiguousarray(logits, dtype=np.float32)
    b = np.ascontiguousarray(bias, dtype=np.float32)
    T, E = l.shape
    idx = np.empty((T, k), dtype=np.int32)
    g = np.empty((T, k), dtype=np.float32)
    s = np.empty((T, E), dtype=np.float32)
    lib().oracle_route(_p(l, ctypes.c_float), _p(b, ctypes.c_float), T, E, k,
                       float(routed_scale), _p(idx, ctypes.c_int32), _p(g, ctypes.c_float),
                       _p(s, ctypes.c_float))
    return idx, g, s


# ------------------------------------------------------------- permutation --

def permute(idx, n_experts: int):
    """Expert-major layout of the routed (token, slot) pairs.

    counts[e]   tokens that selected e
    offsets[e]  exclusive prefix sum of counts (E+1 entries, offsets[E] = T*k)
    row_token[r] token of routed row r; within a segment tokens ascend
    row_of[t,j]  routed row of (t, idx[t,j])
    The shared segment (rows T*k .. T*k+T-1, token order) is implicit.
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)                            # entry t*k + j
    counts = np.bincount(flat, minlength=n_experts).astype(np.int32)
    offsets = np.zeros(n_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    order = np.argsort(flat, kind="stable")           # by expert, then entry (= token) order
    row_token = (order // k).astype(np.int32)
    row_of = np.empty(T * k, dtype=np.int32)
    row_of[order] = np.arange(T * k, dtype=np.int32)
    return counts, offsets, row_token, row_of.reshape(T, k)


# ------------------------------------------------------------ quantisation --

def block_quant(a, block_rows: int, ue8m0: bool = False):
    """e4m3 block quantisation of a [rows, cols] matrix (float32 or bf16 bits).
    ue8m0: power-of-two scales (the UE8M0 variant), else amax / 448.

    -> (codes uint8 [rows, cols], scales fp32 [ceil(rows/block_rows), cols/128])"""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = bf16_to_f32(a)
    a = np.ascontiguousarray(a, dtype=np.float32)
    rows, cols = a.shape
    if cols % 128:
        raise ValueError("cols must be a multiple of 128")
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty(((rows + block_rows - 1) // block_rows, cols // 128), dtype=np.float32)
    fn = lib().oracle_block_quant_ue8m0 if ue8m0 else lib().oracle_block_quant
    fn(_p(a, ctypes.c_float), rows, cols, block_rows, _p(q, ctypes.c_uint8),
       _p(s, ctypes.c_float))
    return q, s


_DEC = None


def dequant(q, scales, block_rows: int) -> np.ndarray:
    """binary64 decode(q) * scale of each block."""
    global _DEC
    if _DEC is None:
        _DEC = e4m3_decode_table()
    q = np.asarray(q, dtype=np.uint8)
    rows, cols = q.shape
    s = np.asarray(scales, dtype=np.float64)
    s_full = np.repeat(np.repeat(s, block_rows, axis=0)[:rows], 128, axis=1)
    return _DEC[q] * s_full


# ----------------------------------------------------------------- experts --

def _silu_mul(g, u):
    return g / (1.0 + np.exp(-g)) * u


def _bf16_of_f64(v) -> np.ndarray:
    # binary64 -> binary32 (round to nearest) -> bf16 (round to nearest even)
    return bf16_from_f32(np.asarray(v, dtype=np.float64).astype(np.float32))


# Two correct evaluations of G and U differ in their accumulation order, so an
# element of H whose e4m3 quantiser input lies at a rounding boundary may take
# either neighbouring code (and, with power-of-two scales, a tile whose amax
# lies at 448 * 2^k either of two scales).  The oracle reports, per output,
# how far such alternative codes could move it; H_FLIP_RHO is the relative
# perturbation of the quantiser input considered.
H_FLIP_RHO = 2.0 ** -14


def h_bf16_ambiguity(Hf, rho: float = H_FLIP_RHO) -> np.ndarray:
    """[n, de] binary64: per element of H in the bf16 precision (Hf: its
    binary64 value before the rounding to bf16), the largest change of its
    bf16 value that a relative perturbation of at most rho could cause: 0
    unless Hf lies within rho of a bf16 rounding boundary, else the gap to
    the bf16 neighbour across that boundary.  Two correct evaluations of G
    and U (accumulated in different orders) may round such an element either
    way, as with the e4m3 codes of the fp8 precisions."""
    Hf = np.asarray(Hf, dtype=np.float64)
    base = bf16_to_f32(_bf16_of_f64(Hf)).astype(np.float64)
    delta = np.zeros_like(base)
    for f in (1.0 + rho, 1.0 - rho):
        alt = bf16_to_f32(_bf16_of_f64(Hf * f)).astype(np.float64)
        delta = np.maximum(delta, np.abs(alt - base))
    return delta


def h_bf16_alternatives(Hf, rho: float = H_FLIP_RHO) -> np.ndarray:
    """[n, de] binary64, signed: for each element of bf16 H within rho of a
    bf16 rounding boundary, the change of its value if it rounded to the
    neighbour across that boundary; 0 elsewhere."""
    Hf = np.asarray(Hf, dtype=np.float64)
    base = bf16_to_f32(_bf16_of_f64(Hf)).astype(np.float64)
    alt = np.zeros_like(base)
    for f in (1.0 + rho, 1.0 - rho):
        d = bf16_to_f32(_bf16_of_f64(Hf * f)).astype(np.float64) - base
        alt = np.where(alt == 0, d, alt)
    return alt


def _ue8m0_exponent(amax):
    m, e = np.frexp(np.asarray(amax, dtype=np.float64))
    return np.maximum(np.where(m > 0.875, e - 8, e - 9), -127)


def h_code_ambiguity(H, hq, hs, ue8m0: bool, rho: float = H_FLIP_RHO) -> np.ndarray:
    """[n, de] binary64: per element of the fp32 H, the largest change of its
    dequantised value that a relative perturbation of at most rho of its
    quantiser input could cause (0 unless the input lies within rho of an
    e4m3 rounding boundary); with power-of-two scales also the change when a
    tile's amax lies within rho of a scale boundary and the scale doubles or
    halves."""
    global _DEC
    if _DEC is None:
        _DEC = e4m3_decode_table()
    H = np.ascontiguousarray(H, dtype=np.float32)
    n, de = H.shape
    base = dequant(hq, hs, 1)
    sc = np.repeat(np.asarray(hs, dtype=np.float64), 128, axis=1)
    amax = np.abs(H).reshape(n, de // 128, 128).max(2)
    if ue8m0:
        x = (H.astype(np.float64) / sc).astype(np.float32)          # exact
    else:
        with np.errstate(divide="ignore"):
            inv = np.where(amax > 0, np.float32(448.0) / amax, np.float32(0.0)).astype(np.float32)
        x = H * np.repeat(inv, 128, axis=1)                          # binary32, as quantised
    delta = np.zeros((n, de))
    for f in (1.0 + rho, 1.0 - rho):
        q = e4m3_encode(x.astype(np.float64) * f)
        delta = np.maximum(delta, np.abs(_DEC[q] * sc - base))
    if ue8m0:
        k = _ue8m0_exponent(amax)
        for f in (1.0 + rho, 1.0 - rho):
            ka = _ue8m0_exponent(amax * f)
            alt = (ka != k) & (amax > 0)
            if alt.any():
                s_alt = np.repeat(np.ldexp(1.0, ka), 128, axis=1)
                q = e4m3_encode(H.astype(np.float64) / s_alt)
                d = np.abs(_DEC[q] * s_alt - base)
                delta = np.where(np.repeat(alt, 128, axis=1), np.maximum(delta, d), delta)
    return delta


def h_code_alternatives(H, hq, hs, ue8m0: bool, rho: float = H_FLIP_RHO) -> np.ndarray:
    """[n, de] binary64, signed: for each element of the fp32 H whose quantiser
    input lies within rho (relative) of an e4m3 rounding boundary, the change
    of its dequantised value if it took the code on the other side of that
    boundary; 0 elsewhere.  These are the other correct H codes; a UE8M0 tile
    whose scale could double or halve is left to h_code_ambiguity's bound."""
    global _DEC
    if _DEC is None:
        _DEC = e4m3_decode_table()
    H = np.ascontiguousarray(H, dtype=np.float32)
    n, de = H.shape
    base = dequant(hq, hs, 1)
    sc = np.repeat(np.asarray(hs, dtype=np.float64), 128, axis=1)
    if ue8m0:
        x = (H.astype(np.float64) / sc).astype(np.float32)
    else:
        amax = np.abs(H).reshape(n, de // 128, 128).max(2)
        with np.errstate(divide="ignore"):
            inv = np.where(amax > 0, np.float32(448.0) / amax, np.float32(0.0)).astype(np.float32)
        x = H * np.repeat(inv, 128, axis=1)
    alt = np.zeros((n, de))
    for f in (1.0 + rho, 1.0 - rho):
        d = _DEC[e4m3_encode(x.astype(np.float64) * f)] * sc - base
        alt = np.where(alt == 0, d, alt)
    return alt


def expert_forward(a_rows, w13, w2, precision: str, a_scales=None, w13_scales=None,
                   w2_scales=None, return_h: bool = False, return_allow: bool = False,
                   return_f64: bool = False, return_alts: bool = False):
    """One gated expert on a block of rows.

    bf16:  a_rows uint16 [n, d], w13 uint16 [2*de, d], w2 uint16 [d, de].
    fp8:   a_rows uint8 codes + a_scales [n, d/128]; w13 codes + w13_scales
           [2*de/128, d/128]; w2 codes + w2_scales [d/128, de/128].
    fp8_ue8m0: as fp8, every scale a power of two; H is requantised the same way.
    -> Y as bf16 bits [n, d] (and H: bf16 bits, or (codes, scales) for fp8;
    return_allow: and [n, d] binary64, how far alternative H codes at e4m3
    rounding boundaries (bf16: alternative bf16 roundings, h_bf16_ambiguity)
    could move Y: sum_i ambiguity_i * |W2[:, i]|; return_f64: (Y in binary64, before its rounding, and that
    allowance), with return_alts also, per row, the [m, d] changes of Y that
    the row's alternative H codes (h_code_alternatives) would make, one row
    per alternative)."""
    n = a_rows.shape[0]
    if precision == "bf16":
        A = bf16_to_f32(a_rows).astype(np.float64)
        W13 = bf16_to_f32(w13).astype(np.float64)
        W2 = bf16_to_f32(w2).astype(np.float64)
        de = W13.shape[0] // 2
        G = A @ W13[:de].T
        U = A @ W13[de:].T
        Hf = _silu_mul(G, U)
        H = _bf16_of_f64(Hf)
        Y = bf16_to_f32(H).astype(np.float64) @ W2.T
        if return_f64:
            allow = h_bf16_ambiguity(Hf) @ np.abs(W2).T
            if return_alts:
                dh = h_bf16_alternatives(Hf)
                alts = []
                for r in range(n):
                    cols = np.nonzero(dh[r])[0]
                    alts.append(dh[r, cols][:, None] * W2[:, cols].T)
                return Y, allow, alts
            return Y, allow
        y = _bf16_of_f64(Y)
        if return_allow:
            return y, h_bf16_ambiguity(Hf) @ np.abs(W2).T
        return (y, H) if return_h else y
    if precision in ("fp8", "fp8_ue8m0"):
        A = dequant(a_rows, a_scales, 1)
        W13 = dequant(w13, w13_scales, 128)
        W2 = dequant(w2, w2_scales, 128)
        de = W13.shape[0] // 2
        G = A @ W13[:de].T
        U = A @ W13[de:].T
        H = _silu_mul(G, U).astype(np.float32)
        ue = precision == "fp8_ue8m0"
        hq, hs = block_quant(H, 1, ue8m0=ue)
        Y = dequant(hq, hs, 1) @ W2.T
        if return_f64:
            allow = h_code_ambiguity(H, hq, hs, ue) @ np.abs(W2).T
            if return_alts:
                dh = h_code_alternatives(H, hq, hs, ue)
                alts = []
                for r in range(n):
                    cols = np.nonzero(dh[r])[0]
                    alts.append(dh[r, cols][:, None] * W2[:, cols].T)
                return Y, allow, alts
            return Y, allow
        y = _bf16_of_f64(Y)
        if return_allow:
            return y, h_code_ambiguity(H, hq, hs, ue) @ np.abs(W2).T
        return (y, (hq, hs)) if return_h else y
    raise ValueError(precision)


# ------------------------------------------------------------------- layer --

def moe_layer(x, w_router, bias, expert, *, n_experts: int, top_k: int, n_shared: int,
              precision: str, routed_scale: float = 1.0, tokens=None, workers: int = 1):
    """Forward of one MoE FFN layer.

    x uint16 [T, d] (bf16 bits); w_router uint16 [E, d]; bias fp32 [E];
    expert(e) -> (w13, w2) as bf16 bits of expert e (e == n_experts is the
    shared expert).  In the fp8 scheme the oracle quantises each expert it
    touches itself (128x128 blocks).
    tokens: indices of the output rows to evaluate (default: all).  Routing,
    permutation and activation quantisation always cover every token.
    workers > 1 evaluates the experts (each on its own, unchanged) on that
    many threads, and the router's logits in as many token chunks; the
    results do not depend on it.

    Returns a dict: logits, scores, idx, gates, counts, offsets, row_token,
    row_of, (fp8) xq, xs, out [len(tokens), d] bf16 bits, tokens."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    T, d = x.shape
    E, k = n_experts, top_k
    logits = router_logits(x, w_router, workers=workers)
    idx, gates, scores = route(logits, bias, k, routed_scale)
    counts, offsets, row_token, row_of = permute(idx, E)
    res = dict(logits=logits, scores=scores, idx=idx, gates=gates, counts=counts,
               offsets=offsets, row_token=row_token, row_of=row_of)
    fp8 = precision in ("fp8", "fp8_ue8m0")
    ue = precision == "fp8_ue8m0"
    if fp8:
        xq, xs = block_quant(x, 1, ue8m0=ue)
        res.update(xq=xq, xs=xs)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    # rows needed per expert: (expert, token) pairs of the evaluated tokens
    need = {}
    for ti, t in enumerate(tokens):
        for j in range(k):
            need.setdefault(int(idx[t, j]), []).append((ti, j))
        if n_shared:
            need.setdefault(E, []).append((ti, k))
    Yt = np.zeros((len(tokens), k + 1, d), dtype=np.float64)
    At = np.zeros((len(tokens), k + 1, d), dtype=np.float64)
    def one_expert(e):
        w13, w2 = expert(e)
        rows = np.array([tokens[ti] for ti, _ in need[e]])
        if fp8:
            w13q, w13s = block_quant(w13, 128, ue8m0=ue)
            w2q, w2s = block_quant(w2, 128, ue8m0=ue)
            y, al = expert_forward(res["xq"][rows], w13q, w2q, precision, res["xs"][rows],
                                   w13s, w2s, return_allow=True)
        else:
            y, al = expert_forward(x[rows], w13, w2, "bf16", return_allow=True)
        return bf16_to_f32(y).astype(np.float64), al

    def store(e, yf, al):
        for n, (ti, j) in enumerate(need[e]):
            Yt[ti, j] = yf[n]
            At[ti, j] = al[n]

    if workers > 1:
        import concurrent.futures as cf
        with cf.ThreadPoolExecutor(int(workers)) as ex:
            for e, (yf, al) in zip(sorted(need), ex.map(one_expert, sorted(need))):
                store(e, yf, al)
    else:
        for e in sorted(need):
            store(e, *one_expert(e))
    g = gates[tokens].astype(np.float64)
    acc = np.einsum("tj,tjd->td", g, Yt[:, :k])
    allow = np.einsum("tj,tjd->td", np.abs(g), At[:, :k])
    if n_shared:
        acc = acc + Yt[:, k]
        allow = allow + At[:, k]
    res["out"] = _bf16_of_f64(acc)
    res["out_f64"] = acc
    # how far alternative H codes at e4m3 rounding boundaries could move out
    res["out_allow"] = allow
    res["tokens"] = tokens
    return res


# ---------------------------------------------------------------- pre-norm --

def rmsnorm(h, gamma, eps: float = 1e-6):
    """Pre-norm of the FFN input (RMSNorm with weight gamma), C core.
    -> (x bf16 bits [T, d], rstd fp32 [T])."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    g = np.ascontiguousarray(gamma, dtype=np.uint16)
    T, d = h.shape
    x = np.empty((T, d), dtype=np.uint16)
    r = np.empty(T, dtype=np.float32)
    lib().oracle_rmsnorm(_p(h, ctypes.c_uint16), _p(g, ctypes.c_uint16), T, d, float(eps),
                         _p(x, ctypes.c_uint16), _p(r, ctypes.c_float))
    return x, r


def moe_layer_prenorm(h, gamma, eps, w_router, bias, expert, **kw):
    """out = h + MoE(RMSNorm(h) * gamma): the FFN block with its pre-norm and
    residual ("DeepSeek-R1" card, "Facts": pre-norm RMSNorm before the MLP).
    The residual is added to the unrounded combine sum in binary64 and the
    block output rounded to bf16 once."""
    x, rstd = rmsnorm(h, gamma, eps)
    tokens = kw.get("tokens")
    res = moe_layer(x, w_router, bias, expert, **kw)
    rows = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    hh = bf16_to_f32(np.asarray(h, dtype=np.uint16)[rows]).astype(np.float64)
    res["moe_out"] = res["out"]
    res["out"] = _bf16_of_f64(hh + res["out_f64"])
    res["x"] = x
    res["rstd"] = rstd
    return res


# ------------------------------------------------------------ dense layer --

def dense_ffn(x, w13, w2, *, precision: str, tokens=None):
    """Dense gated FFN layer (the model's first layers; "DeepSeek-R1" card,
    "Every architecture field": ffns.dense gated, d_ff 18432): one gated MLP
    over every token with the expert numerics of the precision (step 4 of the
    module notes), out = bf16(Y).

    x uint16 [T, d]; w13 uint16 [2*d_ff, d] (gate rows then up rows);
    w2 uint16 [d, d_ff]; tokens: rows to evaluate (default all; activation
    tiles are per row, so a subset quantises exactly as the whole batch).
    Returns dict(out bf16 bits, out_f64, out_allow, tokens, (fp8) xq, xs)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    tokens = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens, dtype=np.int64)
    res = dict(tokens=tokens)
    if precision in ("fp8", "fp8_ue8m0"):
        ue = precision == "fp8_ue8m0"
        xq, xs = block_quant(x[tokens], 1, ue8m0=ue)
        w13q, w13s = block_quant(w13, 128, ue8m0=ue)
        w2q, w2s = block_quant(w2, 128, ue8m0=ue)
        Y, allow, alts = expert_forward(xq, w13q, w2q, precision, xs, w13s, w2s,
                                        return_f64=True, return_alts=True)
        res.update(xq=xq, xs=xs)
    elif precision == "bf16":
        Y, allow, alts = expert_forward(x[tokens], w13, w2, "bf16", return_f64=True,
                                        return_alts=True)
    else:
        raise ValueError(precision)
    res["out_f64"] = Y
    res["out"] = _bf16_of_f64(Y)
    res["out_allow"] = allow
    # per evaluated row: the changes of out_f64 that the row's other correct
    # H codes would make (h_code_alternatives), one row per alternative
    res["out_alts"] = alts
    return res


def dense_ffn_prenorm(h, gamma, eps, w13, w2, *, precision: str, tokens=None):
    """out = bf16(h + FFN(x)), x = RMSNorm(h) * gamma (pre-norm, card "Facts"):
    the residual is added to the binary64 FFN output, one final rounding."""
    x, rstd = rmsnorm(h, gamma, eps)
    res = dense_ffn(x, w13, w2, precision=precision, tokens=tokens)
    hh = bf16_to_f32(np.asarray(h, dtype=np.uint16)[res["tokens"]]).astype(np.float64)
    res["ffn_out"] = res["out"]
    res["out_f64"] = hh + res["out_f64"]
    res["out"] = _bf16_of_f64(res["out_f64"])
    res["x"] = x
    res["rstd"] = rstd
    return res
