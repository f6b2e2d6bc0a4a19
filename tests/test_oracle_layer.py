"""Pins of the oracle's whole layer: the pages' parameter counts, special
cases that reduce to a dense gated MLP written with torch library routines
(identical experts; one token at a time), k = E, and exactness of binary64
sums of e4m3 products."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from moe_inputs import CONFIGS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "deepseek_v3_page_figures.json")


def test_parameter_count_matches_pages():
    """The layer dims reproduce the architecture card's modelled totals
    (669B total, 35.7B active without embeddings) only with three matrices per
    gated expert, 256 + 1 experts of width 2048 and 8 + 1 active."""
    g = json.load(open(GOLDEN))
    d = g["d_model"]["value"]
    E, k = g["n_routed_experts"]["value"], g["n_active_experts"]["value"]
    de, S = g["d_expert"]["value"], g["n_shared_experts"]["value"]
    cfg = CONFIGS["decode"]
    assert (cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_expert, cfg.n_shared) == (d, E, k, de, S)
    m = g["mla"]
    mla = (d * m["q_lora_rank"] + m["q_lora_rank"] * m["heads"] * (m["qk_nope"] + m["qk_rope"])
           + d * (m["kv_lora_rank"] + m["qk_rope"])
           + m["kv_lora_rank"] * m["heads"] * (m["qk_nope"] + m["v_head_dim"])
           + m["heads"] * m["v_head_dim"] * d)
    expert = 3 * d * de
    router = E * d
    nd, nm = g["layout"]["dense_layers"], g["layout"]["moe_layers"]
    dense = 3 * d * g["d_ff_dense"]["value"]
    total = (nd + nm) * mla + nd * dense + nm * ((E + S) * expert + router)
    active = (nd + nm) * mla + nd * dense + nm * ((k + S) * expert + router)
    pf = g["modelled_params_without_embeddings"]
    assert round(total / 1e9) == pf["total_B"]
    assert round(active / 1e9, 1) == pf["active_B"]
    ae = g["active_experts_per_layer"]
    assert (k + S, E + S, S) == (ae["active"], ae["total"], ae["shared"])
    two_matrix = 2 * d * de
    assert round(two_matrix / 1e6, 2) == g["activated_ffn_params_B"]["per_expert_M"]
    n_active = nm * (k + S) + nd * (E + S)
    assert round(n_active * two_matrix / 1e9, 2) == g["activated_ffn_params_B"]["value"]


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _dense_expert_bf16(x, w13, w2):
    """Gated MLP in binary64 with torch ops; H and Y stored as bf16."""
    de = w13.shape[0] // 2
    A = x.double()
    G = A @ w13[:de].double().T
    U = A @ w13[de:].double().T
    H = (F.silu(G) * U).float().bfloat16()
    return (H.double() @ w2.double().T).float().bfloat16()


def _tq(a, block_rows):
    """Independent blockwise quantise-dequantise with torch's float8 cast."""
    a = a.float()
    rows, cols = a.shape
    out = torch.empty(rows, cols, dtype=torch.float64)
    for r0 in range(0, rows, block_rows):
        for c0 in range(0, cols, 128):
            t = a[r0:r0 + block_rows, c0:c0 + 128]
            amax = t.abs().max()
            if amax == 0:
                out[r0:r0 + block_rows, c0:c0 + 128] = 0
                continue
            sc = (amax / 448.0).float()
            inv = (torch.tensor(448.0) / amax).float()
            q = (t * inv).to(torch.float8_e4m3fn)
            out[r0:r0 + block_rows, c0:c0 + 128] = q.double() * sc.double()
    return out


def _dense_expert_fp8(x, w13, w2):
    de = w13.shape[0] // 2
    A = _tq(x, 1)
    W13 = _tq(w13, 128)
    W2 = _tq(w2, 128)
    G = A @ W13[:de].T
    U = A @ W13[de:].T
    H = (F.silu(G) * U).float()
    return (_tq(H, 1) @ W2.T).float().bfloat16()


def _run_oracle(cfg, inp, tokens=None):
    return oracle.moe_layer(
        _u16(inp["x"]), _u16(inp["w_router"]), inp["bias"].numpy(),
        lambda e: (_u16(inp["w13"][e]), _u16(inp["w2"][e])),
        n_experts=cfg.n_experts, top_k=cfg.top_k, n_shared=cfg.n_shared,
        precision=cfg.precision, routed_scale=cfg.routed_scale, tokens=tokens)


def _close_bf16(out_u16, ref_u16):
    """True where out is within one bf16 step of ref; a floor at 2^-20 of the
    reference RMS absorbs sign flips of values that cancel to almost zero."""
    a = oracle.bf16_to_f32(out_u16).astype(np.float64)
    b = oracle.bf16_to_f32(ref_u16).astype(np.float64)
    rms = np.sqrt(np.mean(b * b))
    return np.abs(a - b) <= np.maximum(2.0 ** -7 * np.abs(b), 2.0 ** -20 * rms)


@pytest.mark.parametrize("precision", ["bf16", "fp8"])
def test_identical_experts_reduce_to_dense(precision):
    cfg = CONFIGS["tiny"].with_(precision=precision, T=48)
    inp = make_inputs(cfg, seed=3, identical_experts=True)
    res = _run_oracle(cfg, inp)
    dense = _dense_expert_bf16 if precision == "bf16" else _dense_expert_fp8
    y_r = dense(inp["x"], inp["w13"][0], inp["w2"][0]).double()
    y_s = dense(inp["x"], inp["w13"][cfg.n_experts], inp["w2"][cfg.n_experts]).double()
    ref = _u16((y_r + y_s).float().bfloat16())
    # the gates sum to 1 up to a few binary32 roundings, so out is at most one
    # bf16 step away; sums of two bf16 values often sit exactly on a rounding
    # tie, which that tiny perturbation may break either way
    assert _close_bf16(res["out"], ref).all()
    assert (res["out"] != ref).mean() < 0.05


@pytest.mark.parametrize("precision", ["bf16", "fp8"])
def test_token_by_token_matches_permuted_layer(precision):
    """Per token, out = sum_j g_j * Expert_{idx_j}(x) + Shared(x), evaluated
    without any permutation."""
    cfg = CONFIGS["tiny"].with_(precision=precision, T=6, d_model=256, n_experts=8, top_k=3,
                                d_expert=128)
    inp = make_inputs(cfg, seed=4)
    res = _run_oracle(cfg, inp)
    dense = _dense_expert_bf16 if precision == "bf16" else _dense_expert_fp8
    E, k = cfg.n_experts, cfg.top_k
    for t in range(cfg.T):
        xt = inp["x"][t:t + 1]
        acc = torch.zeros(1, cfg.d_model, dtype=torch.float64)
        for j in range(k):
            e = int(res["idx"][t, j])
            acc += float(res["gates"][t, j]) * dense(xt, inp["w13"][e], inp["w2"][e]).double()
        acc += dense(xt, inp["w13"][E], inp["w2"][E]).double()
        ref = _u16(acc.float().bfloat16())
        assert _close_bf16(res["out"][t:t + 1], ref).all()


def test_k_equals_E_all_experts_active():
    cfg = CONFIGS["tiny"].with_(T=8, top_k=16)
    inp = make_inputs(cfg, seed=5)
    res = _run_oracle(cfg, inp)
    assert (np.sort(res["idx"], 1) == np.arange(16)).all()
    assert list(res["counts"]) == [8] * 16
    s = res["scores"].astype(np.float64)
    sj = np.take_along_axis(s, res["idx"], 1)
    assert np.allclose(res["gates"], sj / s.sum(1, keepdims=True), rtol=1e-6)


def test_sampled_tokens_equal_full_rows():
    cfg = CONFIGS["tiny"].with_(T=40)
    inp = make_inputs(cfg, seed=6)
    full = _run_oracle(cfg, inp)
    part = _run_oracle(cfg, inp, tokens=[3, 17, 39])
    assert np.array_equal(part["out"], full["out"][[3, 17, 39]])


def test_fp64_block_partials_of_e4m3_are_exact():
    """Every e4m3 x e4m3 product has at most 8 significant bits and 128 of them
    span less than 2^43, so binary64 sums them exactly in any order."""
    rng = np.random.default_rng(9)
    table = oracle.e4m3_decode_table()
    finite = np.array([c for c in range(256) if not np.isnan(table[c])], np.uint8)
    qa = rng.choice(finite, (4, 128))
    qw = rng.choice(finite, (3, 128))
    ones_a = np.ones((4, 1), np.float32)
    ones_w = np.ones((1, 1), np.float32)
    P = oracle.dequant(qa, ones_a, 1) @ oracle.dequant(qw, ones_w, 128).T
    for i in range(4):
        for j in range(3):
            exact = sum(Fraction(float(table[a])) * Fraction(float(table[b]))
                        for a, b in zip(qa[i], qw[j]))
            assert Fraction(float(P[i, j])) == exact
