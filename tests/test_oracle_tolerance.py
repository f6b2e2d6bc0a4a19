"""Pins of the oracle's bound on alternative H codes (oracle.h_code_ambiguity),
which widens the max-abs output tolerance of the fp8 precisions: checked on
constructed tiles whose quantiser inputs are known exactly."""
import numpy as np
import pytest

import oracle
from moe_inputs import DENSE_CONFIGS, make_dense_inputs


def _tile(vals, amax_at=0, amax=448.0):
    """One 1x128 row whose quantiser input equals `vals` exactly (scale 1)."""
    h = np.zeros((1, 128), np.float32)
    h[0, amax_at] = amax
    h[0, 1:1 + len(vals)] = vals
    return h


@pytest.mark.parametrize("ue8m0", [False, True])
def test_zero_away_from_boundaries(ue8m0):
    # amax 448 gives scale 1 in both variants; codes exactly representable
    h = _tile([1.0, -1.125, 3.5, 0.015625, -240.0])
    q, s = oracle.block_quant(h, 1, ue8m0=ue8m0)
    assert s[0, 0] == 1.0
    d = oracle.h_code_ambiguity(h, q, s, ue8m0)
    assert not d.any()


@pytest.mark.parametrize("ue8m0", [False, True])
def test_one_step_at_a_rounding_midpoint(ue8m0):
    # 1.0625 lies half way between the e4m3 values 1.0 and 1.125 (ties to even
    # gives 1.0); a perturbation either way reaches 1.125: one step of 0.125
    h = _tile([1.0625, 1.03125])
    q, s = oracle.block_quant(h, 1, ue8m0=ue8m0)
    d = oracle.h_code_ambiguity(h, q, s, ue8m0)
    assert d[0, 1] == 0.125
    assert d[0, 2] == 0.0                       # a quarter step from the boundary
    assert np.count_nonzero(d) == 1


def test_scale_boundary_of_power_of_two_tiles():
    # amax exactly 448 * 2^3: scale 2^3, and the next binary32 value up takes
    # 2^4, so every element may be requantised at the doubled scale
    h = _tile([9.0, 1.0], amax=448.0 * 8)
    q, s = oracle.block_quant(h, 1, ue8m0=True)
    assert s[0, 0] == 8.0
    d = oracle.h_code_ambiguity(h, q, s, True)
    # 9 = 1.125 * 8 (exact at scale 8); at scale 16, 9/16 = 0.5625 is an e4m3
    # value too, so 9 stays exact; 1 = 0.125 * 8 and 1/16 = 0.0625 both exact
    assert d[0, 1] == 0.0 and d[0, 2] == 0.0
    h2 = _tile([9.5], amax=448.0 * 8)
    q2, s2 = oracle.block_quant(h2, 1, ue8m0=True)
    d2 = oracle.h_code_ambiguity(h2, q2, s2, True)
    # 9.5/8 = 1.1875 rounds to 1.25 (ties to even between 1.125 and 1.25) ->
    # 10; 9.5/16 = 0.59375 rounds to 0.625 (ties to even) -> 10: same value,
    # but the midpoint itself is ambiguous at scale 8: 9 or 10
    assert d2[0, 1] == 1.0


def test_layer_allowance_is_small_in_every_precision():
    """A handful of H elements per row sit near a rounding boundary (bf16 or
    e4m3), so the allowance stays well below the output scale."""
    from moe_inputs import CONFIGS, make_inputs
    import torch
    u16 = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    for prec in ("bf16", "fp8", "fp8_ue8m0"):
        cfg = CONFIGS["tiny"].with_(precision=prec, T=8)
        inp = make_inputs(cfg, seed=2)
        res = oracle.moe_layer(u16(inp["x"]), u16(inp["w_router"]), inp["bias"].numpy(),
                               lambda e: (u16(inp["w13"][e]), u16(inp["w2"][e])),
                               n_experts=cfg.n_experts, top_k=cfg.top_k, n_shared=cfg.n_shared,
                               precision=prec)
        out = oracle.bf16_to_f32(res["out"]).astype(np.float64)
        rms = np.sqrt(np.mean(out ** 2))
        # a handful of boundary elements per row: well below the output scale
        assert res["out_allow"].max() < 0.1 * rms


# ------------------------------------------- alternative codes (signed) --

def test_alternatives_are_the_neighbouring_codes():
    """h_code_alternatives gives, for each element whose quantiser input is
    within rho of a rounding boundary, the other code's change: it is the
    adjacent e4m3 value on the far side of that boundary, the boundary lies
    within rho of the input, and its magnitude is h_code_ambiguity's bound
    (with fp32 scales that bound has no other source)."""
    rng = np.random.default_rng(31)
    H = (rng.standard_normal((16, 256)) * np.exp(rng.uniform(-3, 3, (16, 1)))).astype(np.float32)
    rho = 2.0 ** -7  # wide, so that many elements have an alternative
    hq, hs = oracle.block_quant(H, 1)
    alt = oracle.h_code_alternatives(H, hq, hs, False, rho=rho)
    amb = oracle.h_code_ambiguity(H, hq, hs, False, rho=rho)
    assert np.array_equal(np.abs(alt), amb)
    assert (alt != 0).sum() > 50
    table = oracle.e4m3_decode_table()
    finite = np.sort(np.unique(np.abs(table[np.isfinite(table)])))
    sc = np.repeat(hs, 128, axis=1)
    cur = table[hq]
    amax = np.abs(H).reshape(16, 2, 128).max(2)
    x = H * np.repeat((np.float32(448.0) / amax).astype(np.float32), 128, axis=1)
    for r, c in zip(*np.nonzero(alt)):
        other = (cur[r, c] * sc[r, c] + alt[r, c]) / sc[r, c]
        a, b = sorted((abs(cur[r, c]), abs(other)))
        i = np.searchsorted(finite, a)
        assert finite[i] == a and finite[i + 1] == b          # adjacent magnitudes
        assert np.sign(other) * np.sign(cur[r, c]) >= 0       # same side of zero
        mid = (a + b) / 2
        assert abs(abs(float(x[r, c])) - mid) <= rho * abs(float(x[r, c])) * 1.0000001


def test_nearest_correct_output_takes_only_explaining_alternatives():
    """The checker: an output made with the oracle's largest alternative code
    is recognised (its distance to the nearest correct output drops to the
    bf16 rounding level); a planted error of the same size that no
    alternative explains is not absorbed."""
    import torch
    from _gpu_util import nearest_correct_output, out_error
    cfg = DENSE_CONFIGS["dense_tiny"].with_(T=24)
    inp = make_dense_inputs(cfg, seed=32)
    u = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    res = oracle.dense_ffn(u(inp["x"]), u(inp["w13"]), u(inp["w2"]), precision="fp8")
    cand = [(np.linalg.norm(v), r, i) for r, a in enumerate(res["out_alts"]) for i, v in enumerate(a)]
    assert cand, "no alternative codes in this sample"
    _, r, i = max(cand)
    v = res["out_alts"][r][i]
    as_bf16 = lambda a: torch.from_numpy(
        oracle.bf16_from_f32(a.astype(np.float32)).view(np.int16)).view(torch.bfloat16)
    flipped = res["out_f64"].copy()
    flipped[r] += v
    got = as_bf16(flipped)
    want, taken, cands = nearest_correct_output(got, res["out_f64"], res["out_alts"])
    assert taken >= 1 and cands >= taken
    rel_plain = out_error(got, res["out"])[0]
    rel_near = out_error(got, want)[0]
    assert rel_near < rel_plain / 4
    # the same change moved to other columns is no alternative
    bad = res["out_f64"].copy()
    bad[r] += np.roll(v, 17)
    got_bad = as_bf16(bad)
    want_bad, _, _ = nearest_correct_output(got_bad, res["out_f64"], res["out_alts"])
    assert out_error(got_bad, want_bad)[0] > 0.5 * out_error(got_bad, res["out"])[0]


def test_nearest_correct_output_without_alternatives_is_the_oracles():
    """With no alternatives the nearest correct output is the oracle's own
    bf16 output, bit for bit."""
    import torch
    from _gpu_util import nearest_correct_output
    cfg = DENSE_CONFIGS["dense_tiny"].with_(T=12, precision="bf16")
    inp = make_dense_inputs(cfg, seed=33)
    u = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    res = oracle.dense_ffn(u(inp["x"]), u(inp["w13"]), u(inp["w2"]), precision="bf16")
    none = [np.zeros((0, cfg.d_model))] * cfg.T
    got = torch.from_numpy(res["out"].view(np.int16)).view(torch.bfloat16)
    want, taken, cands = nearest_correct_output(got, res["out_f64"], none)
    assert taken == 0 and cands == 0 and np.array_equal(want, res["out"])


def _bf16_round_torch(v):
    """bf16 value of binary64 v via torch (binary32 first, as the oracle and
    the GPU round): an implementation independent of the oracle's codec."""
    import torch
    return torch.from_numpy(np.asarray(v, dtype=np.float64).astype(np.float32)).to(
        torch.bfloat16).to(torch.float64).numpy()


def test_bf16_h_ambiguity_is_the_neighbour_gap_at_boundaries():
    """h_bf16_ambiguity: exactly the gap to the bf16 neighbour for values
    within rho of a rounding boundary (midpoints of adjacent bf16 values),
    0 for values well inside a rounding interval; checked against torch's
    bf16 rounding of the perturbed values.  h_bf16_alternatives gives the
    signed change to that neighbour."""
    rng = np.random.default_rng(35)
    rho = 2.0 ** -14
    lo = _bf16_round_torch(np.exp(rng.uniform(-6, 6, 400)) * rng.choice([-1, 1], 400))
    step = 2.0 ** (np.floor(np.log2(np.abs(lo))) - 7)
    hi = lo + np.sign(lo) * step                        # the next bf16 magnitude
    mid = (lo + hi) / 2                                  # rounding boundary
    near = mid * (1 + rng.uniform(-0.5, 0.5, 400) * rho)   # within rho of it
    inside = lo + np.sign(lo) * step / 4                 # a quarter step from lo
    H = np.stack([near, inside])
    amb = oracle.h_bf16_ambiguity(H, rho)
    alt = oracle.h_bf16_alternatives(H, rho)
    base = _bf16_round_torch(H)
    brute = np.maximum(np.abs(_bf16_round_torch(H * (1 + rho)) - base),
                       np.abs(_bf16_round_torch(H * (1 - rho)) - base))
    assert np.array_equal(amb, brute)
    assert np.allclose(amb[0], step, rtol=0, atol=0)     # every boundary value: one step
    assert np.all(amb[1] == 0) and np.all(alt[1] == 0)
    other = base[0] + alt[0]                             # the neighbour across the boundary
    assert np.all(np.isin(other, np.stack([lo, hi]))) and np.all(other != base[0])


def test_bf16_layer_allowance_covers_a_planted_flip():
    """The bf16 expert's allowance bounds the output change of any one H
    element taking its other rounding: plant the flip of the in-band element
    with the largest effect and compare row by row."""
    cfg = DENSE_CONFIGS["dense_tiny"].with_(T=16, precision="bf16")
    inp = make_dense_inputs(cfg, seed=36)
    import torch
    u = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    x, w13, w2 = u(inp["x"]), u(inp["w13"]), u(inp["w2"])
    Y, allow, alts = oracle.expert_forward(x, w13, w2, "bf16", return_f64=True, return_alts=True)
    assert sum(len(a) for a in alts) > 0, "no element near a bf16 boundary in this sample"
    for r, a in enumerate(alts):
        for v in a:
            assert np.all(np.abs(v) <= allow[r] * (1 + 1e-12))
def test_ue8m0_alternatives_are_adjacent_codes_within_the_bound():
    """With power-of-two scales the code-level alternatives are again the
    neighbouring e4m3 values across a boundary, and never exceed
    h_code_ambiguity, which also covers whole-tile scale changes."""
    rng = np.random.default_rng(34)
    H = (rng.standard_normal((16, 256)) * np.exp(rng.uniform(-3, 3, (16, 1)))).astype(np.float32)
    rho = 2.0 ** -7
    hq, hs = oracle.block_quant(H, 1, ue8m0=True)
    alt = oracle.h_code_alternatives(H, hq, hs, True, rho=rho)
    amb = oracle.h_code_ambiguity(H, hq, hs, True, rho=rho)
    assert (alt != 0).sum() > 50
    assert np.all(np.abs(alt) <= amb)
    table = oracle.e4m3_decode_table()
    finite = np.sort(np.unique(np.abs(table[np.isfinite(table)])))
    sc = np.repeat(hs, 128, axis=1)
    cur = table[hq]
    for r, c in zip(*np.nonzero(alt)):
        other = (cur[r, c] * sc[r, c] + alt[r, c]) / sc[r, c]
        a, b = sorted((abs(cur[r, c]), abs(other)))
        i = np.searchsorted(finite, a)
        assert finite[i] == a and finite[i + 1] == b
