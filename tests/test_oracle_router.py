"""Pins of the oracle's router: logit order and error bound, brute-force
top-k, gate invariants, and the routing-only role of the bias ("DeepSeek v3
and R1 Model Architecture", "Local Balanced Routing to Experts")."""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def test_logits_sequential_order():
    """1 + 2^-24 ties to 1 under round-to-nearest-even, so a left-to-right
    sum stays at 1.0; any other order that first adds the small terms gives
    1 + 8 * 2^-24."""
    x = np.array([[1.0] + [2.0 ** -24] * 8], dtype=np.float32)
    w = np.ones((1, 9), dtype=np.float32)
    l = oracle.router_logits(_bf16(x), _bf16(w))
    assert l[0, 0] == 1.0
    xr = x[:, ::-1].copy()
    l2 = oracle.router_logits(_bf16(xr), _bf16(w))
    assert l2[0, 0] == np.float32(1.0 + 8 * 2.0 ** -24)


def test_logits_error_bound_vs_exact():
    rng = np.random.default_rng(5)
    T, E, d = 4, 6, 512
    x = _bf16(rng.normal(0, 1, (T, d)))
    w = _bf16(rng.normal(0, 1 / np.sqrt(d), (E, d)))
    l = oracle.router_logits(x, w)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    wf = oracle.bf16_to_f32(w).astype(np.float64)
    u = 2.0 ** -24
    for t in range(T):
        for e in range(E):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xf[t], wf[e]))
            bound = d * u / (1 - d * u) * float(np.sum(np.abs(xf[t] * wf[e])))
            assert abs(float(Fraction(float(l[t, e])) - exact)) <= bound


def _topk_bruteforce(sel, k):
    """Subset S of size k such that every member beats every non-member under
    (value desc, index asc); among all size-k subsets it is the unique one."""
    E = len(sel)
    hits = []
    for S in itertools.combinations(range(E), k):
        ok = all((sel[i] > sel[j]) or (sel[i] == sel[j] and i < j)
                 for i in S for j in range(E) if j not in S)
        if ok:
            hits.append(S)
    assert len(hits) == 1
    S = hits[0]
    # the selected set also has the maximal exact sum
    best = max(sum(Fraction(float(sel[i])) for i in C) for C in itertools.combinations(range(E), k))
    assert sum(Fraction(float(sel[i])) for i in S) == best
    return sorted(S, key=lambda i: (-sel[i], i))


@pytest.mark.parametrize("case", ["random", "ties", "allequal", "bias"])
def test_topk_bruteforce_E16_k4(case):
    rng = np.random.default_rng({"random": 0, "ties": 1, "allequal": 2, "bias": 3}[case])
    T, E, k = 60, 16, 4
    if case == "random":
        logits = rng.normal(0, 1, (T, E)).astype(np.float32)
        bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    elif case == "ties":     # few distinct values: many exact ties
        logits = rng.integers(-2, 3, (T, E)).astype(np.float32) * 0.25
        bias = np.zeros(E, np.float32)
    elif case == "allequal":
        logits = np.zeros((T, E), np.float32)
        bias = np.zeros(E, np.float32)
    else:
        logits = rng.normal(0, 0.5, (T, E)).astype(np.float32)
        bias = (rng.integers(0, 2, E) * 0.7).astype(np.float32)
    idx, g, s = oracle.route(logits, bias, k)
    sel = (s + bias[None, :]).astype(np.float32)
    for t in range(T):
        assert list(idx[t]) == _topk_bruteforce(list(sel[t]), k)
    if case == "allequal":
        assert (idx == np.arange(k)[None, :]).all()


def test_gates_normalised_and_bias_free():
    rng = np.random.default_rng(7)
    T, E, k = 200, 32, 6
    logits = rng.normal(0, 1, (T, E)).astype(np.float32)
    bias = rng.uniform(-0.3, 0.3, E).astype(np.float32)
    for rs in (1.0, 2.5):
        idx, g, s = oracle.route(logits, bias, k, rs)
        # scores are the sigmoid of the logits, untouched by the bias
        assert np.array_equal(s, oracle.sigmoid(logits))
        sj = np.take_along_axis(s, idx, 1).astype(np.float64)
        ref = sj / sj.sum(1, keepdims=True) * rs
        # S carries k-1 roundings, then one division and one multiply
        assert np.all(np.abs(g - ref) <= (k + 2) * 2.0 ** -24 * np.abs(ref))
        assert np.all(np.abs(g.astype(np.float64).sum(1) - rs) <= 4 * k * np.spacing(np.float32(rs)))
    # a huge bias on expert 3 forces its selection, but its gate stays its affinity share
    b2 = bias.copy()
    b2[3] = 10.0
    idx2, g2, s2 = oracle.route(logits, b2, k)
    assert (idx2[:, 0] == 3).all()
    sj = np.take_along_axis(s2, idx2, 1).astype(np.float64)
    assert np.allclose(g2, sj / sj.sum(1, keepdims=True), rtol=1e-6)
    # zero bias: selection = top-k of the affinities
    idx0, _, s0 = oracle.route(logits, np.zeros(E, np.float32), k)
    for t in range(20):
        order = sorted(range(E), key=lambda e: (-s0[t, e], e))[:k]
        assert list(idx0[t]) == order


def test_k_equals_E_selects_all():
    rng = np.random.default_rng(8)
    logits = rng.normal(0, 1, (10, 16)).astype(np.float32)
    idx, g, s = oracle.route(logits, np.zeros(16, np.float32), 16)
    assert all(sorted(r) == list(range(16)) for r in idx)
