"""CPU checks of the C ABI: the library loads without a GPU, exports every
function include/moe_fwd.h declares, and rejects bad arguments on the host
(before touching CUDA) with the documented codes."""
import ctypes
import os
import re

import pytest

import sparse_moe_transformer_fwd_b200 as moe
from sparse_moe_transformer_fwd_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_fwd.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_header_functions_exported():
    names = _declared_functions()
    assert len(names) >= 10, names
    L = moe.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing
    assert sorted(N.EXPORTS) == names


def _shape(**kw):
    s = dict(T=64, d_model=7168, n_experts=256, top_k=8, d_expert=2048, n_shared=1,
             routed_scale=1.0, precision="fp8")
    s.update(kw)
    return moe.make_shape(**s)


def test_workspace_size_and_bad_shapes():
    assert moe.moe_workspace_size(_shape()) > 64 * 7168 * 9
    for bad in (dict(d_model=7000), dict(d_model=384), dict(d_expert=100), dict(top_k=0),
                dict(top_k=33), dict(top_k=300), dict(n_shared=2), dict(n_experts=1024),
                dict(precision=7), dict(T=-1)):
        assert moe.lib().moe_workspace_size(ctypes.byref(_shape(**bad))) == 0, bad
        assert moe.moe_last_error()


FAKE = ctypes.c_void_p(0x7F0000001000)       # never dereferenced on the host
MISALIGNED = ctypes.c_void_p(0x7F0000001004)


def _call_forward(shape, ws_bytes, x=FAKE, ws=FAKE):
    L = moe.lib()
    return L.moe_forward(ctypes.byref(shape), x, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                         ws, ws_bytes, None)


def test_host_side_errors_return_codes():
    s = _shape()
    need = moe.moe_workspace_size(s)
    assert _call_forward(_shape(d_model=100), need) == N.MOE_ERR_INVALID_ARG
    assert _call_forward(s, need - 1) == N.MOE_ERR_WORKSPACE
    assert "needs" in moe.moe_last_error()
    assert _call_forward(s, need, ws=ctypes.c_void_p(0x7F0000001010)) == N.MOE_ERR_INVALID_ARG
    assert _call_forward(s, need, x=MISALIGNED) == N.MOE_ERR_INVALID_ARG
    assert "aligned" in moe.moe_last_error()
    assert _call_forward(s, need, x=None) == N.MOE_ERR_INVALID_ARG
    L = moe.lib()
    assert L.fp8_block_quant(FAKE, 10, 100, 100, 1, 0, FAKE, FAKE, None) == N.MOE_ERR_INVALID_ARG
    assert L.fp8_block_quant(FAKE, 10, 128, 128, 64, 0, FAKE, FAKE, None) == N.MOE_ERR_INVALID_ARG
    assert L.fp8_block_quant(FAKE, 100, 128, 128, 128, 1, FAKE, FAKE, None) == N.MOE_ERR_INVALID_ARG
    assert L.fp8_block_quant(FAKE, 128, 128, 128, 1, 1, FAKE, FAKE, None) == N.MOE_ERR_INVALID_ARG
    assert L.fp8_block_quant(FAKE, 0, 128, 128, 1, 0, FAKE, FAKE, None) == N.MOE_OK
    assert L.moe_pack_tiles(FAKE, 100, 128, FAKE, None) == N.MOE_ERR_INVALID_ARG
    assert L.moe_pack_tiles(FAKE, 128, 96, FAKE, None) == N.MOE_ERR_INVALID_ARG


def test_empty_batch_enqueues_nothing():
    s = _shape(T=0)
    assert _call_forward(s, moe.moe_workspace_size(s)) == N.MOE_OK
    assert moe.moe_last_launch_count() == 0
    assert moe.moe_last_launch_names() == []
    assert moe.lib().moe_last_launch_name(0) is None


def test_binding_rejects_cpu_tensors():
    import torch
    s = _shape(T=4, d_model=256, n_experts=16, top_k=4, d_expert=128)
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moe.moe_route(s, x, x, x, x, x, torch.zeros(16, dtype=torch.uint8))


def _dense(**kw):
    a = dict(T=64, d_model=7168, d_ff=18432, precision="fp8")
    a.update(kw)
    return moe.make_dense_shape(**a)


def test_dense_workspace_and_host_errors():
    """The dense layer's workspace (split-K partials only up to 256 tokens)
    and its host-side argument checks; nothing here launches a kernel."""
    L = moe.lib()
    small, big = moe.moe_dense_workspace_size(_dense()), moe.moe_dense_workspace_size(_dense(T=257))
    assert small >= 64 * 7168 * 8 * 4 + 64 * (7168 + 18432)   # partials + x and H codes
    assert big < 257 * (7168 + 18432) * 2 + 257 * 4 * 256      # no partials past 256 tokens
    for bad in (dict(d_model=7000), dict(d_model=384), dict(d_ff=100), dict(precision=7),
                dict(T=-1)):
        assert L.moe_dense_workspace_size(ctypes.byref(_dense(**bad))) == 0, bad
    s = _dense()
    need = moe.moe_dense_workspace_size(s)
    call = lambda shape, nbytes, x=FAKE, w13s=FAKE: L.moe_dense_ffn(
        ctypes.byref(shape), x, FAKE, w13s, FAKE, FAKE, FAKE, FAKE, nbytes, None)
    assert call(s, need - 1) == N.MOE_ERR_WORKSPACE
    assert call(s, need, x=MISALIGNED) == N.MOE_ERR_INVALID_ARG
    assert call(s, need, w13s=None) == N.MOE_ERR_INVALID_ARG      # e4m3 needs scales
    assert L.moe_dense_ffn_prenorm(ctypes.byref(s), FAKE, None, ctypes.c_float(1e-6), FAKE, FAKE,
                                   FAKE, FAKE, FAKE, FAKE, need, None) == N.MOE_ERR_INVALID_ARG
    e = _dense(T=0)
    assert call(e, moe.moe_dense_workspace_size(e)) == N.MOE_OK
    assert moe.moe_last_launch_count() == 0


def test_weight_layout_is_declared_and_checked():
    """The shape declares the weights' layout: row-major (0, the value of a
    zero-initialised shape) or tiled (1); any other value is rejected on the
    host before anything is enqueued, for the MoE and the dense layer."""
    assert N.MOE_LAYOUT_ROWMAJOR == 0 and N.MOE_LAYOUT_TILED == 1
    assert moe.make_shape(64, 7168, 256, 8, 2048).weight_layout == N.MOE_LAYOUT_TILED
    zero = N.MoeShape()
    assert zero.weight_layout == N.MOE_LAYOUT_ROWMAJOR
    for lay in (N.MOE_LAYOUT_ROWMAJOR, N.MOE_LAYOUT_TILED):
        assert moe.moe_workspace_size(_shape(weight_layout=lay)) > 0
        assert moe.moe_dense_workspace_size(_dense(weight_layout=lay)) > 0
    for bad in (2, -1, 7):
        s = _shape(weight_layout=bad)
        assert moe.lib().moe_workspace_size(ctypes.byref(s)) == 0
        assert "weight_layout" in moe.moe_last_error()
        assert _call_forward(s, 1 << 30) == N.MOE_ERR_INVALID_ARG
        assert moe.lib().moe_dense_workspace_size(ctypes.byref(_dense(weight_layout=bad))) == 0


def test_workspace_layout_regions():
    """moe_workspace_layout: every region starts on a 256-byte boundary,
    regions follow one another without overlap in the order listed, sized
    for the shape, and the total is moe_workspace_size."""
    for kw in (dict(), dict(precision="bf16"), dict(T=16384), dict(T=1, n_experts=16, top_k=4,
                                                                    d_model=512, d_expert=256)):
        s = _shape(**kw)
        o = moe.moe_workspace_layout(s)
        assert o["total"] == moe.moe_workspace_size(s)
        T, E, k, d, de = s.T, s.n_experts, s.top_k, s.d_model, s.d_expert
        Rs = T * (k + s.n_shared)
        es = 2 if s.precision == N.MOE_BF16 else 1
        need = {"scores": T * E * 4, "topk_idx": T * k * 4, "topk_w": T * k * 4,
                "counts": E * 4, "offsets": (E + 1) * 4, "row_token": T * k * 4,
                "row_of": T * k * 4, "a": Rs * d * es, "h": Rs * de * es, "y": Rs * d * 2}
        if es == 1:
            need.update(a_scales=Rs * (d // 128) * 4, h_scales=Rs * (de // 128) * 4)
        names = sorted(need, key=lambda n: o[n])
        for a, b in zip(names, names[1:]):
            assert o[a] % 256 == 0 and o[a] + need[a] <= o[b], (a, b)
        assert o[names[-1]] + need[names[-1]] <= o["total"]
    with pytest.raises(moe.MoeError):
        moe.moe_workspace_layout(_shape(d_model=100))
