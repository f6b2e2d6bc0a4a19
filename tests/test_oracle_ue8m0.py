"""Pins of the oracle's UE8M0 variant of the blockwise e4m3 quantiser (scales
rounded up to a power of two, "DeepSeek-R1" (aguasto.com), "Quantization":
blockwise FP8; the power-of-two scale is the reading of the next scope row).

The oracle computes k from frexp; these tests check it against other
characterisations: the least power of two that bounds amax / 448 (exact
rationals), torch's float8 cast for the codes, and a dense torch layer whose
exponent comes from log2 with an exact correction."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from moe_inputs import CONFIGS, make_inputs


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _least_pow2_exponent(amax: float) -> int:
    """Least integer k >= -127 (the smallest UE8M0 exponent) with
    amax <= 448 * 2^k, from log2 then corrected with exact rational
    comparisons."""
    a = Fraction(amax)
    k = math.ceil(math.log2(amax / 448.0))
    while a > 448 * Fraction(2) ** k:
        k += 1
    while a <= 448 * Fraction(2) ** (k - 1):
        k -= 1
    return max(k, -127)


def _tiles(rng, rows, cols):
    """Rows of very different magnitude, bf16-representable, incl. subnormals."""
    a = rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-140, 120, (rows, 1)))
    return torch.from_numpy(a.astype(np.float32)).bfloat16().float().numpy()


@pytest.mark.parametrize("block_rows", [1, 128])
def test_scale_is_least_power_of_two_bound(block_rows):
    rng = np.random.default_rng(21 + block_rows)
    rows = 300 if block_rows == 1 else 260
    a = _tiles(rng, rows, 256)
    a[3, :128] = 0.0
    q, s = oracle.block_quant(a, block_rows, ue8m0=True)
    for rb in range(s.shape[0]):
        for kb in range(s.shape[1]):
            tile = a[rb * block_rows:(rb + 1) * block_rows, kb * 128:(kb + 1) * 128]
            amax = float(np.abs(tile).max())
            sc = float(s[rb, kb])
            m, e = math.frexp(sc)
            assert m == 0.5, sc                       # a power of two
            if amax == 0.0:
                assert sc == 1.0
                continue
            assert sc == 2.0 ** _least_pow2_exponent(amax)
            assert 0 <= e - 1 + 127 <= 254            # representable as UE8M0


@pytest.mark.parametrize("j", [-120, -20, 0, 5, 100])
def test_boundaries_of_the_rounding(j):
    """amax exactly 448 * 2^j takes 2^j; the next binary32 value above takes
    2^(j+1); the one below keeps 2^j."""
    base = np.float32(448.0 * 2.0 ** j)
    for amax, want in ((base, j), (np.nextafter(base, np.float32(np.inf)), j + 1),
                       (np.nextafter(base, np.float32(0)), j)):
        t = np.zeros((1, 128), np.float32)
        t[0, 7] = amax
        t[0, 8] = -amax / 3
        _, s = oracle.block_quant(t, 1, ue8m0=True)
        assert s[0, 0] == np.float32(2.0 ** want)


def test_codes_are_torch_float8_of_exact_quotient():
    rng = np.random.default_rng(7)
    a = _tiles(rng, 64, 512)
    q, s = oracle.block_quant(a, 1, ue8m0=True)
    table = oracle.e4m3_decode_table()
    for r in range(64):
        for kb in range(4):
            tile = a[r, kb * 128:(kb + 1) * 128].astype(np.float64)
            sc = float(s[r, kb])
            if np.abs(tile).max() == 0:                   # zero tile (incl. -0.0): +0 codes
                assert sc == 1.0 and not q[r, kb * 128:(kb + 1) * 128].any()
                continue
            exact = (tile / sc).astype(np.float32)        # power-of-two quotient: exact
            assert np.array_equal(exact.astype(np.float64) * sc, tile)
            ref = torch.from_numpy(exact).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(ref, q[r, kb * 128:(kb + 1) * 128])
            dec = np.abs(table[q[r, kb * 128:(kb + 1) * 128]])
            assert dec.max() <= 448.0
            if sc > 2.0 ** -127:
                # above the exponent floor the largest quotient lies in
                # (224, 448], so it rounds into [224, 448]
                assert dec.max() >= 224.0


def test_exponent_floor():
    """Tiles below 448 * 2^-128 keep the smallest UE8M0 scale 2^-127; their
    codes still equal the float8 cast of the (exact) quotient."""
    t = np.zeros((1, 128), np.float32)
    t[0, :4] = [2.0 ** -130, -3 * 2.0 ** -133, 2.0 ** -133, 1.5 * 2.0 ** -129]
    q, s = oracle.block_quant(t, 1, ue8m0=True)
    assert s[0, 0] == np.float32(2.0 ** -127)
    ref = torch.from_numpy((t.astype(np.float64) * 2.0 ** 127).astype(np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ref, q)
    assert q[0, 0] == 0x20          # 2^-3 exactly


def test_zero_tile_and_extremes():
    t = np.zeros((2, 256), np.float32)
    t[1, :128] = 3.3895313892515355e38          # largest finite bf16
    t[1, 128] = 9.183549615799121e-41            # smallest bf16 subnormal
    q, s = oracle.block_quant(t, 1, ue8m0=True)
    assert s[0, 0] == 1.0 and s[0, 1] == 1.0 and not q[0].any()
    assert s[1, 0] == np.float32(2.0 ** _least_pow2_exponent(3.3895313892515355e38))
    assert s[1, 1] == np.float32(2.0 ** _least_pow2_exponent(9.183549615799121e-41))


# ------------------------------------------------------------------ layer --

def _tq_pow2(a, block_rows):
    """Independent quantise-dequantise: log2-derived exponent, torch cast."""
    a = a.float()
    rows, cols = a.shape
    out = torch.empty(rows, cols, dtype=torch.float64)
    for r0 in range(0, rows, block_rows):
        for c0 in range(0, cols, 128):
            t = a[r0:r0 + block_rows, c0:c0 + 128]
            amax = float(t.abs().max())
            if amax == 0:
                out[r0:r0 + block_rows, c0:c0 + 128] = 0
                continue
            k = _least_pow2_exponent(amax)
            q = (t.double() * 2.0 ** -k).float().to(torch.float8_e4m3fn)
            out[r0:r0 + block_rows, c0:c0 + 128] = q.double() * 2.0 ** k
    return out


def _dense_expert_ue8m0(x, w13, w2):
    de = w13.shape[0] // 2
    A = _tq_pow2(x, 1)
    W13 = _tq_pow2(w13, 128)
    W2 = _tq_pow2(w2, 128)
    G = A @ W13[:de].T
    U = A @ W13[de:].T
    H = (F.silu(G) * U).float()
    return (_tq_pow2(H, 1) @ W2.T).float().bfloat16()


def _close_bf16(out_u16, ref_u16):
    a = oracle.bf16_to_f32(out_u16).astype(np.float64)
    b = oracle.bf16_to_f32(ref_u16).astype(np.float64)
    rms = np.sqrt(np.mean(b * b))
    return np.abs(a - b) <= np.maximum(2.0 ** -7 * np.abs(b), 2.0 ** -20 * rms)


def test_layer_token_by_token_matches_dense_ue8m0():
    """out[t] = sum_j g_j Expert_{idx_j}(x_t) + Shared(x_t) with every tensor
    quantised by the independent power-of-two quantiser above."""
    cfg = CONFIGS["tiny"].with_(precision="fp8_ue8m0", T=6, d_model=256, n_experts=8,
                                top_k=3, d_expert=128)
    inp = make_inputs(cfg, seed=4)
    res = oracle.moe_layer(
        _u16(inp["x"]), _u16(inp["w_router"]), inp["bias"].numpy(),
        lambda e: (_u16(inp["w13"][e]), _u16(inp["w2"][e])),
        n_experts=cfg.n_experts, top_k=cfg.top_k, n_shared=cfg.n_shared,
        precision=cfg.precision)
    E, k = cfg.n_experts, cfg.top_k
    for t in range(cfg.T):
        xt = inp["x"][t:t + 1]
        acc = torch.zeros(1, cfg.d_model, dtype=torch.float64)
        for j in range(k):
            e = int(res["idx"][t, j])
            acc += float(res["gates"][t, j]) * _dense_expert_ue8m0(xt, inp["w13"][e],
                                                                   inp["w2"][e]).double()
        acc += _dense_expert_ue8m0(xt, inp["w13"][E], inp["w2"][E]).double()
        assert _close_bf16(res["out"][t:t + 1], _u16(acc.float().bfloat16())).all()


def test_ue8m0_differs_from_fp32_scales():
    """The two readings are different quantisers: on the same activations the
    codes differ wherever amax / 448 is not already a power of two."""
    cfg = CONFIGS["tiny"].with_(T=16)
    x = _u16(make_inputs(cfg, seed=1)["x"])
    q1, s1 = oracle.block_quant(x, 1)
    q2, s2 = oracle.block_quant(x, 1, ue8m0=True)
    assert np.all(s2 >= s1)
    assert (q1 != q2).any()
