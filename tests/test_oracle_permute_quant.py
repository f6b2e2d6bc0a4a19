"""Pins of the oracle's permutation (invariants of a stable expert-major
layout) and of its blockwise e4m3 quantiser (error bound, amax -> 448,
agreement with torch's float8_e4m3fn cast of the scaled values)."""
import numpy as np
import pytest
import torch

import oracle


def _random_idx(rng, T, E, k):
    return np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k", [(1, 16, 4), (129, 16, 4), (300, 256, 8), (64, 8, 8)])
def test_permute_invariants(T, E, k):
    rng = np.random.default_rng(T + E)
    idx = _random_idx(rng, T, E, k)
    counts, offsets, row_token, row_of = oracle.permute(idx, E)
    assert counts.sum() == T * k and offsets[0] == 0 and offsets[E] == T * k
    assert np.array_equal(np.diff(offsets), counts)
    seg = np.searchsorted(offsets, np.arange(T * k), side="right") - 1
    # every routed row belongs to a segment whose expert the token selected
    for r in range(T * k):
        assert seg[r] in idx[row_token[r]]
    # tokens strictly ascend inside each segment (stable, no duplicates)
    for e in range(E):
        toks = row_token[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(toks) > 0)
        assert set(toks) == {t for t in range(T) if e in idx[t]}
    # row_of inverts row_token; each token lands in exactly k distinct rows
    assert np.array_equal(np.sort(row_of.reshape(-1)), np.arange(T * k))
    for t in range(T):
        for j in range(k):
            r = row_of[t, j]
            assert row_token[r] == t and seg[r] == idx[t, j]


def test_permute_empty_and_all_on_one():
    idx = np.zeros((50, 1), np.int32) + 3
    counts, offsets, row_token, row_of = oracle.permute(idx, 8)
    assert list(counts) == [0, 0, 0, 50, 0, 0, 0, 0]
    assert list(row_token) == list(range(50)) and list(row_of[:, 0]) == list(range(50))


def _quantum(code_vals):
    """Spacing of the e4m3 grid at each decoded magnitude (binade quantum)."""
    a = np.abs(code_vals)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return 2.0 ** (e - 3)


@pytest.mark.parametrize("block_rows", [1, 128])
def test_block_quant_bound_and_amax(block_rows):
    rng = np.random.default_rng(11 + block_rows)
    rows, cols = 260, 384            # ragged last row-block for 128-row blocks
    a = (rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-6, 3, (rows, 1)))).astype(np.float32)
    a[5, 128:256] = 0.0              # an all-zero 1x128 tile
    q, s = oracle.block_quant(a, block_rows)
    nrb = (rows + block_rows - 1) // block_rows
    assert s.shape == (nrb, cols // 128)
    table = oracle.e4m3_decode_table()
    for rb in range(nrb):
        for kb in range(cols // 128):
            tile = a[rb * block_rows:(rb + 1) * block_rows, kb * 128:(kb + 1) * 128]
            qt = q[rb * block_rows:(rb + 1) * block_rows, kb * 128:(kb + 1) * 128]
            amax = np.abs(tile).max()
            sc = s[rb, kb]
            if amax == 0:
                assert sc == 1.0 and np.all(qt == 0)
                continue
            assert sc == np.float32(amax) / np.float32(448.0)
            dec = table[qt]
            # the amax element encodes to +-448
            i = np.unravel_index(np.argmax(np.abs(tile)), tile.shape)
            assert abs(dec[i]) == 448.0
            # |x - dec*scale| <= half a grid step, in units of the scale (plus the
            # binary32 rounding of x * inv, at most 2^-24 relative)
            err = np.abs(tile.astype(np.float64) / float(sc) - dec)
            assert np.all(err <= 0.5 * _quantum(dec) + 2.0 ** -22 * np.abs(dec) + 1e-12)
    # codes equal torch's float8 cast of the scaled values
    for rb in range(min(nrb, 3)):
        tile = a[rb * block_rows:(rb + 1) * block_rows, :128]
        amax = np.abs(tile).max()
        inv = np.float32(448.0) / np.float32(amax)
        ref = torch.from_numpy((tile * inv).astype(np.float32)).to(torch.float8_e4m3fn).view(
            torch.uint8).numpy()
        assert np.array_equal(ref, q[rb * block_rows:(rb + 1) * block_rows, :128])


def test_dequant_layout():
    q = np.full((256, 256), 0x38, np.uint8)     # e4m3 1.0
    s = np.array([[1.0, 2.0], [3.0, 4.0]], np.float32)
    d = oracle.dequant(q, s, 128)
    assert d[0, 0] == 1 and d[0, 200] == 2 and d[200, 0] == 3 and d[255, 255] == 4
    s1 = np.arange(512, dtype=np.float32).reshape(256, 2)
    d1 = oracle.dequant(q, s1, 1)
    assert d1[7, 3] == s1[7, 0] and d1[7, 130] == s1[7, 1]
