"""Helpers shared by the GPU parity tests: tensor conversions, running the
oracle on the same inputs, and the output tolerance.

Tolerance of a bf16 output against the oracle's bf16-rounded output:
relative L2 <= 1e-3, and max |diff| <= 1e-2 * RMS(oracle) beyond one bf16
step of the oracle value.  The step allowance is the storage quantum: two
correct evaluations whose binary32 / binary64 sums straddle a bf16 rounding
boundary store values one step apart, and a step is |v|/256..|v|/128, which
is larger than 1e-2 * RMS wherever |v| > 1.28 * RMS.  Without it no bf16
output could meet the max-abs bound.  In the fp8 precisions the max bound also
allows, per output, the oracle's bound on how far alternative e4m3 codes of H
could move it (H elements whose quantiser input lies at a rounding boundary,
oracle.h_code_ambiguity): two correct evaluations of G and U may round such
an element either way, and one code step of a large H element moves every
output of its row by up to one step times |W2|.  Where such flips are common
enough to move the relative L2 as well (the dense layer: all 18432 H elements
of a row feed each of its outputs with weight 1), the comparison is with the
correct output nearest to the GPU's: the oracle's, with the row's
alternative H codes that explain the difference (nearest_correct_output)."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle

REL_L2 = 1e-3
MAX_ABS_RMS = 1e-2


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_u16(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def untile(a: np.ndarray, rows: int, row_bytes: int) -> np.ndarray:
    """Tiled layout (128 x 128-byte tiles, include/moe_fwd.h) -> row-major
    uint8 [rows, row_bytes]."""
    t = np.ascontiguousarray(a).view(np.uint8).reshape(rows // 128, row_bytes // 128, 128, 128)
    return t.transpose(0, 2, 1, 3).reshape(rows, row_bytes)


def bf16_step(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |v| (8 significant bits)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def out_error(got_bf16: torch.Tensor, want_u16: np.ndarray, allow=None):
    """-> (relative L2, max |diff| / RMS, max (|diff| - one bf16 step - allow)+ / RMS)."""
    got = got_bf16.detach().float().cpu().numpy().astype(np.float64)
    want = oracle.bf16_to_f32(want_u16).astype(np.float64).reshape(got.shape)
    diff = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300)
    rms = max(np.sqrt(np.mean(want ** 2)), 1e-300)
    slack = bf16_step(want)
    if allow is not None:
        slack = slack + np.asarray(allow, dtype=np.float64).reshape(got.shape)
    excess = np.maximum(diff - slack, 0.0)
    return rel, diff.max() / rms, excess.max() / rms


def _log(what, rel, mx, ex, **extra):
    path = os.environ.get("MOE_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", ""), "what": what,
                                "rel_l2": rel, "max_over_rms": mx,
                                "beyond_allowance_over_rms": ex, **extra}) + "\n")


def assert_out_close(got_bf16, want_u16, what="", allow=None, **extra):
    rel, mx, ex = out_error(got_bf16, want_u16, allow)
    _log(what, rel, mx, ex, **extra)
    assert rel <= REL_L2 and ex <= MAX_ABS_RMS, \
        f"{what}: rel_l2={rel:.3e} max/rms={mx:.3e} beyond-one-step/rms={ex:.3e}"
    return rel, mx, ex


# An alternative is taken only when the GPU output's projection on it exceeds
# half its length (the point past which it brings the output closer) by
# Z_NOISE standard deviations of that projection under bf16 rounding noise
# alone.
Z_NOISE = 4.0


def nearest_correct_output(got_bf16, out_f64, alts, z: float = Z_NOISE):
    """Several outputs are correct when elements of H sit at e4m3 rounding
    boundaries: the oracle's, and the oracle's with any of those elements on
    the other code (oracle.h_code_alternatives; alts[r] lists the changes of
    row r, one per alternative).  Per row, alternative V (largest first) is
    taken when the residual r = got - current output satisfies
        r . V - |V|^2 / 2  >  z * sqrt(sum_i V_i^2 sigma_i^2),
    sigma_i^2 = step_i^2 / 12 being the variance of the bf16 rounding of the
    GPU's element i (step_i the bf16 spacing at it).  The left side is half
    the drop in squared distance that taking V gives; the right side is z
    standard deviations of r . V when got differs from the current output
    by rounding alone.  So an alternative is taken only where it explains
    the GPU's output beyond rounding noise.
    -> (bf16 bits of that output, rounded as the oracle rounds, number of
    alternatives taken, number of candidates)."""
    got = got_bf16.detach().float().cpu().numpy().astype(np.float64)
    adj = np.array(out_f64, dtype=np.float64).reshape(got.shape).copy()
    sig2 = bf16_step(got) ** 2 / 12.0
    taken = cands = 0
    for r, V in enumerate(alts):
        V = np.asarray(V, dtype=np.float64)
        if V.size == 0:
            continue
        cands += V.shape[0]
        res = got[r] - adj[r]
        for i in np.argsort(-np.linalg.norm(V, axis=1)):
            v = V[i]
            vv = v @ v
            if vv == 0.0:
                continue
            if res @ v - vv / 2 > z * np.sqrt((v * v) @ sig2[r]):
                res = res - v
                adj[r] += v
                taken += 1
    return oracle.bf16_from_f32(adj.astype(np.float32)), taken, cands


# Bound on the alternatives taken, against the candidates (elements of H whose
# quantiser input lies within 2^-14, relative, of an e4m3 rounding boundary).
# The GPU's binary32 G and U differ from the oracle's binary64 ones by about
# 2^-18 relative, so an element in the band takes the other code with a
# probability of about 2^-18 / 2^-14 = 1/16; the bound allows four times that
# and a few more.
def max_alternatives(cands: int) -> int:
    return 4 + cands // 4


def assert_close_to_correct(got_bf16, res, what=""):
    """The output tolerance against the nearest correct output (above), with
    the max bound's allowance for the alternatives not taken; the number of
    alternatives taken stays within max_alternatives of the candidates."""
    want, taken, cands = nearest_correct_output(got_bf16, res["out_f64"], res["out_alts"])
    oracle_out = res["out"] if "out" in res else oracle.bf16_from_f32(
        np.asarray(res["out_f64"], dtype=np.float64).astype(np.float32))
    plain = out_error(got_bf16, oracle_out, res["out_allow"])
    out = assert_out_close(got_bf16, want, what, allow=res["out_allow"],
                           alternatives_taken=taken, alternatives_in_band=cands,
                           rel_l2_before_alternatives=plain[0])
    assert taken <= max_alternatives(cands), f"{what}: {taken} alternatives of {cands} taken"
    return out


# host threads the oracle may use for its independent experts (each expert's
# evaluation stays single-threaded; results do not depend on the count)
ORACLE_WORKERS = max(1, min(len(os.sched_getaffinity(0)), 16))


def oracle_layer(cfg, inp, tokens=None, expert=None, workers=ORACLE_WORKERS):
    """Oracle forward of the layer on the tokens listed (default all).  Tokens
    of an MoE layer are independent, so a subset is evaluated as its own batch."""
    x = inp["x"] if tokens is None else inp["x"][torch.as_tensor(tokens, device=inp["x"].device)]
    if expert is None:
        expert = lambda e: (u16(inp["w13"][e]), u16(inp["w2"][e]))
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        return oracle.moe_layer(u16(x), u16(inp["w_router"]), inp["bias"].detach().cpu().numpy(),
                                expert, n_experts=cfg.n_experts, top_k=cfg.top_k,
                                n_shared=cfg.n_shared, precision=cfg.precision,
                                routed_scale=cfg.routed_scale, workers=workers)
