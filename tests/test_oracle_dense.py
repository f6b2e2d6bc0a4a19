"""Pins of the oracle's dense gated FFN layer (the model's first layers,
"DeepSeek-R1" card, "Every architecture field": ffns.dense gated, d_ff
18432): against a dense gated MLP written with torch library routines and an
independent blockwise quantiser (torch's float8 cast), against the MoE
layer's shared-expert path, and the pre-norm block's residual."""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import CONFIGS, DENSE_CONFIGS, make_dense_inputs, make_inputs, make_residual
from test_oracle_layer import _close_bf16, _dense_expert_bf16, _dense_expert_fp8
from test_oracle_ue8m0 import _dense_expert_ue8m0


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


_TORCH_DENSE = {"bf16": _dense_expert_bf16, "fp8": _dense_expert_fp8,
                "fp8_ue8m0": _dense_expert_ue8m0}


@pytest.mark.parametrize("precision", ["bf16", "fp8", "fp8_ue8m0"])
def test_dense_matches_torch_gated_mlp(precision):
    """Odd sizes: d_ff = 640 (5 K blocks in the down projection), 37 tokens."""
    cfg = DENSE_CONFIGS["dense_tiny"].with_(T=37, d_model=256, d_ff=640, precision=precision)
    inp = make_dense_inputs(cfg, seed=5)
    res = oracle.dense_ffn(_u16(inp["x"]), _u16(inp["w13"]), _u16(inp["w2"]),
                           precision=precision)
    ref = _u16(_TORCH_DENSE[precision](inp["x"], inp["w13"], inp["w2"]))
    # both sides round one binary64 value to bf16; their sums differ in order
    assert _close_bf16(res["out"], ref).all()
    assert (res["out"] != ref).mean() < 0.02
    assert res["out"].shape == (37, 256)


@pytest.mark.parametrize("precision", ["bf16", "fp8"])
def test_dense_equals_moe_shared_path(precision):
    """A MoE layer whose routed experts are all zero reduces to its shared
    expert: its output equals the dense layer's on the shared weights."""
    cfg = CONFIGS["tiny"].with_(precision=precision, T=20)
    inp = make_inputs(cfg, seed=6)
    E = cfg.n_experts
    zero13 = np.zeros_like(_u16(inp["w13"][0]))
    zero2 = np.zeros_like(_u16(inp["w2"][0]))
    ex = lambda e: (_u16(inp["w13"][e]), _u16(inp["w2"][e])) if e == E else (zero13, zero2)
    moe = oracle.moe_layer(_u16(inp["x"]), _u16(inp["w_router"]), inp["bias"].numpy(), ex,
                           n_experts=E, top_k=cfg.top_k, n_shared=1, precision=precision)
    dense = oracle.dense_ffn(_u16(inp["x"]), _u16(inp["w13"][E]), _u16(inp["w2"][E]),
                             precision=precision)
    assert np.array_equal(moe["out"], dense["out"])


def test_dense_sampled_tokens_equal_full_rows():
    cfg = DENSE_CONFIGS["dense_tiny"].with_(T=40)
    inp = make_dense_inputs(cfg, seed=7)
    args = (_u16(inp["x"]), _u16(inp["w13"]), _u16(inp["w2"]))
    full = oracle.dense_ffn(*args, precision="fp8")
    tok = np.array([0, 7, 39, 12])
    part = oracle.dense_ffn(*args, precision="fp8", tokens=tok)
    assert np.array_equal(part["out"], full["out"][tok])
    assert np.array_equal(part["out_allow"], full["out_allow"][tok])


def test_dense_prenorm_adds_residual_once():
    cfg = DENSE_CONFIGS["dense_tiny"].with_(T=16)
    inp = make_dense_inputs(cfg, seed=8)
    h, g = make_residual(cfg, seed=8)
    blk = oracle.dense_ffn_prenorm(_u16(h), _u16(g), 1e-6, _u16(inp["w13"]), _u16(inp["w2"]),
                                   precision="fp8")
    # independent path: torch pre-norm, torch gated MLP in binary64, + h
    hf = h.double()
    rstd = torch.from_numpy(blk["rstd"]).double()
    x = ((h.float() * rstd.float()[:, None]) * g.float()[None, :]).bfloat16()
    assert np.array_equal(blk["x"], _u16(x))
    y = _dense_expert_fp8(x, inp["w13"], inp["w2"]).double()
    # the block rounds h + Y once; the reference rounds Y to bf16 first, and
    # that double rounding can land one bf16 step (relative spacing <= 2^-7)
    # away, plus the half step of Y's own rounding (relative <= 2^-8)
    ref = (hf + y).float().bfloat16().double().numpy()
    got = oracle.bf16_to_f32(blk["out"]).astype(np.float64)
    step = np.abs(ref) * 2.0 ** -7 + np.abs(y.numpy()) * 2.0 ** -8
    assert np.all(np.abs(got - ref) <= step)
    assert (got != ref).mean() < 0.1
