"""Pins of the oracle's pre-norm (RMSNorm before the MLP, "DeepSeek-R1" card,
"Facts"): rstd against its binary64 definition, the summation order, the
element rounding, and the block's residual."""
import numpy as np
import torch

import oracle
from moe_inputs import CONFIGS, make_inputs, make_residual


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_rstd_close_to_definition():
    cfg = CONFIGS["tiny"].with_(T=64, d_model=7168)
    h, g = make_residual(cfg, seed=1)
    x, r = oracle.rmsnorm(_u16(h), _u16(g), 1e-6)
    hf = h.double().numpy()
    ref = 1.0 / np.sqrt((hf * hf).mean(1) + 1e-6)
    # binary32 sum of 7168 squares: relative error well below 1e-5
    assert np.max(np.abs(r / ref - 1)) < 1e-5


def test_rstd_summation_order():
    """d = 32, h_0 = 4096 (square 2^24) and h_1..h_31 = 1: a left-to-right sum
    drops every +1 (ties to even) and gives 2^24; the butterfly of the spec
    meets lane 0 with partial sums 1, 2, 4, 8, 16 and gives 2^24 + 30."""
    h = np.array([[4096.0] + [1.0] * 31], dtype=np.float32)
    g = np.ones(32, dtype=np.float32)
    bf = lambda a: torch.from_numpy(a).bfloat16().view(torch.int16).numpy().view(np.uint16)
    _, r = oracle.rmsnorm(bf(h), bf(g), 0.0)
    S = np.float32(2.0 ** 24 + 30)
    expect = np.float32(1.0) / np.sqrt(S / np.float32(32.0))
    assert r[0] == expect
    assert r[0] != np.float32(1.0) / np.sqrt(np.float32(2.0 ** 24) / np.float32(32.0))


def test_x_is_bf16_of_scaled_product():
    cfg = CONFIGS["tiny"].with_(T=16)
    h, g = make_residual(cfg, seed=2)
    x, r = oracle.rmsnorm(_u16(h), _u16(g), 1e-6)
    ref = ((h.float() * torch.from_numpy(r)[:, None]) * g.float()[None, :]).bfloat16()
    assert np.array_equal(x, _u16(ref))


def test_block_adds_residual_once():
    cfg = CONFIGS["tiny"].with_(T=12)
    inp = make_inputs(cfg, seed=3)
    h, g = make_residual(cfg, seed=3)
    ex = lambda e: (_u16(inp["w13"][e]), _u16(inp["w2"][e]))
    args = dict(n_experts=cfg.n_experts, top_k=cfg.top_k, n_shared=1, precision="bf16")
    blk = oracle.moe_layer_prenorm(_u16(h), _u16(g), 1e-6, _u16(inp["w_router"]),
                                   inp["bias"].numpy(), ex, **args)
    x, _ = oracle.rmsnorm(_u16(h), _u16(g), 1e-6)
    plain = oracle.moe_layer(x, _u16(inp["w_router"]), inp["bias"].numpy(), ex, **args)
    assert np.array_equal(blk["idx"], plain["idx"])
    ref = oracle.bf16_from_f32((h.double().numpy() + plain["out_f64"]).astype(np.float32))
    assert np.array_equal(blk["out"], ref)
