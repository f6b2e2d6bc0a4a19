"""Pins of the oracle's number codecs and its sigmoid against things other
than itself: torch's float8_e4m3fn and bfloat16 casts (library routines),
a brute-force nearest-value search over the e4m3 value set, and binary64
math.exp / 1/(1+exp) with ulp bounds."""
import math

import numpy as np
import pytest
import torch

import oracle


def _f32_patterns():
    """Every binary32 whose top 12 mantissa bits are arbitrary and whose low 11
    bits take one of a set of edge patterns, over the binades 2^-14 .. 2^10,
    both signs: covers every e4m3 rounding boundary and its neighbours."""
    hi = np.arange(1 << 12, dtype=np.uint32) << 11
    lows = np.array([0, 1, 2, 0x3FF, 0x400, 0x401, 0x7FE, 0x7FF], dtype=np.uint32)
    mant = (hi[:, None] | lows[None, :]).reshape(-1)
    exps = np.arange(127 - 14, 127 + 11, dtype=np.uint32)
    bits = (exps[:, None] << 23 | mant[None, :]).reshape(-1)
    bits = np.concatenate([bits, bits | 0x80000000, np.array([0, 0x80000000], np.uint32)])
    return bits.view(np.float32)


def test_e4m3_decode_matches_torch():
    table = oracle.e4m3_decode_table()
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(table))
    assert nan.sum() == 2                    # S.1111.111 only: no infinities
    assert np.array_equal(table[~nan], ref[~nan])
    assert table[0x7E] == 448.0 and table[0xFE] == -448.0
    assert table[0x01] == 2.0 ** -9 and table[0x08] == 2.0 ** -6


def test_e4m3_encode_matches_torch_in_range():
    v = _f32_patterns()
    v = v[np.abs(v) < 464.0]                 # torch turns >= 464 into NaN (no saturation)
    ours = oracle.e4m3_encode(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, (v[bad[:5]], ours[bad[:5]], ref[bad[:5]])


def test_e4m3_encode_saturates():
    v = np.array([448.0, 463.9, 464.0, 480.0, 1e6, 3e38, -464.0, -1e30], dtype=np.float32)
    ours = oracle.e4m3_encode(v)
    assert list(ours) == [0x7E] * 6 + [0xFE] * 2


def test_e4m3_encode_is_nearest_ties_even_bruteforce():
    """Brute force: nearest of the 253 finite values; on a tie the even code."""
    table = oracle.e4m3_decode_table()
    finite = [c for c in range(256) if not np.isnan(table[c])]
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.uniform(-448, 448, 2000), rng.uniform(-2, 2, 2000),
                        rng.uniform(-2 ** -6, 2 ** -6, 2000)]).astype(np.float32)
    # exact midpoints between neighbouring positive values
    pos = sorted({table[c] for c in finite if table[c] >= 0})
    mids = np.array([(a + b) / 2 for a, b in zip(pos[:-1], pos[1:])], dtype=np.float32)
    v = np.concatenate([v, mids, -mids])
    ours = oracle.e4m3_encode(v)
    for x, c in zip(v.astype(np.float64), ours):
        dist = [(abs(table[f] - x), f) for f in finite]
        best = min(d for d, _ in dist)
        cands = [f for d, f in dist if d == best]
        if len(cands) > 1:   # tie between two values (or +-0): the even mantissa
            cands = [f for f in cands if (f & 1) == 0] or cands
        assert table[c] in [table[f] for f in cands], (x, c, cands)


def test_bf16_round_matches_torch():
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    lows = np.array([0, 1, 0x7FFF, 0x8000, 0x8001, 0xFFFF], dtype=np.uint32)
    bits = (hi[:, None] | lows[None, :]).reshape(-1)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    ours = oracle.bf16_from_f32(f)
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(oracle.bf16_to_f32(ours),
                          torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def _ulp32(x):
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 23)


def test_exp_cw_within_3ulp():
    rng = np.random.default_rng(2)
    ys = np.concatenate([np.linspace(-87, 87, 20001), rng.uniform(-87, 87, 20000),
                         [0.0, 1.0, -1.0, math.log(2), 0.5 * math.log(2)]]).astype(np.float32)
    got = np.array([oracle.exp_cw(float(y)) for y in ys])
    ref = np.exp(ys.astype(np.float64))
    err = np.abs(got - ref) / _ulp32(ref)
    assert err.max() <= 3.0, err.max()
    assert oracle.exp_cw(0.0) == 1.0


def test_sigmoid_within_4ulp():
    rng = np.random.default_rng(3)
    l = np.concatenate([np.linspace(-20, 20, 40001), rng.normal(0, 0.5, 40000),
                        rng.uniform(-90, 90, 2000)]).astype(np.float32)
    got = oracle.sigmoid(l).astype(np.float64)
    lc = np.clip(l.astype(np.float64), -87, 87)
    ref = 1.0 / (1.0 + np.exp(-lc))
    err = np.abs(got - ref) / _ulp32(ref)
    assert err.max() <= 4.0, err.max()
    assert oracle.sigmoid(np.float32([0.0]))[0] == 0.5
    # symmetry sigma(-l) = 1 - sigma(l) up to rounding
    s1 = oracle.sigmoid(l[:1000]).astype(np.float64)
    s2 = oracle.sigmoid(-l[:1000]).astype(np.float64)
    assert np.max(np.abs(s1 + s2 - 1.0)) < 4 * 2.0 ** -24 * 2
