"""The benchmark's roofline arithmetic, checked on the CPU: the algorithmic
bytes of the dominant GEMM agree with the DRAM bytes ncu counted for it
(profiles/roofline_traffic.json), the dense layer's bound is the roof with
the longer floor, and the traffic record is only used for the sources it
was taken on."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from moe_inputs import CONFIGS, DENSE_CONFIGS  # noqa: E402

RECORD = os.path.join(ROOT, "profiles", "roofline_traffic.json")
PEAKS = {"hbm_gbs": 6545.3, "bf16_tflops": 1667.2, "bf16_tflops_sustained": 1396.9}


def test_gate_up_algorithmic_bytes_match_measured_dram():
    """Decode: 154 routed experts were touched (102 of 256 got no token) plus
    the shared one; ncu read the gate/up GEMM's weights once, so the two
    counts agree within 0.5 %.  155 touched experts give the bench's
    4,557,405,184 algorithmic bytes exactly."""
    rec = json.load(open(RECORD))
    measured = rec["workloads"]["decode"]["grouped_gemm_gate_up"]["traffic_bytes_per_launch"]
    alg = bench.algorithmic_bytes_gemm1(CONFIGS["decode"], touched=155)
    assert alg == 4557405184
    assert abs(alg - measured) / measured < 0.005


def test_moe_roofline_bound_follows_the_longer_floor():
    """The MoE arm's bound is the roof with the longer floor at the measured
    peaks: HBM for decode and prefill (weights dominate), tensor for the
    skewed T=16384 batch (8.66 TFLOP of gate/up against ~8.9 GB) and for the
    bf16 T=8192 batch; frac = achieved / peak, recomputable from the line."""
    dec = bench.moe_roofline(CONFIGS["decode"], 155, 0.6664, PEAKS, "measured")
    assert dec["bound"] == "hbm" and dec["unit"] == "GB/s"
    assert dec["achieved"] == pytest.approx(4557405184 / 0.6664e-3 / 1e9, rel=1e-4)
    pre = bench.moe_roofline(CONFIGS["prefill"], 257, 2.15, PEAKS, "measured")
    assert pre["bound"] == "hbm"
    skew = bench.moe_roofline(CONFIGS["skew"], 257, 6.37, PEAKS, "measured")
    assert skew["bound"] == "tensor" and skew["unit"] == "TFLOP/s"
    flops = 2.0 * 16384 * 9 * 4096 * 7168
    assert skew["algorithmic_flops"] == flops
    assert skew["peak"] == pytest.approx(2 * PEAKS["bf16_tflops"])
    assert skew["achieved"] == pytest.approx(flops / 6.37e-3 / 1e12, rel=1e-4)
    assert skew["frac"] == pytest.approx(skew["achieved"] / skew["peak"], rel=1e-3)
    b16 = bench.moe_roofline(CONFIGS["bf16"], 257, 5.6, PEAKS, "measured")
    assert b16["bound"] == "tensor" and b16["peak"] == pytest.approx(PEAKS["bf16_tflops"])


def test_layer_floor():
    """Whole-layer floor: the longer of (touched experts' three matrices and
    scales + x in + out) / HBM and (both GEMMs' FLOPs) / tensor peak."""
    c = CONFIGS["skew"]
    f = bench.layer_floor(c, 257, 12.3, PEAKS)
    w = 257 * (3 * 2048 * 7168 + 4 * (32 * 56 + 56 * 16))
    t_hbm = (w + 16384 * 7168 * 4) / (PEAKS["hbm_gbs"] * 1e9) * 1e3
    t_tc = 2.0 * 16384 * 9 * 3 * 2048 * 7168 / (2 * PEAKS["bf16_tflops"] * 1e12) * 1e3
    assert f["bound"] == "tensor"
    assert f["floor_ms"] == pytest.approx(max(t_hbm, t_tc), abs=1e-4)
    assert f["frac"] == pytest.approx(max(t_hbm, t_tc) / 12.3, abs=1e-4)
    assert bench.layer_floor(CONFIGS["decode"], 155, 1.05, PEAKS)["bound"] == "hbm"


def test_dense_roofline_bounds_and_bytes():
    dec = bench.dense_roofline(DENSE_CONFIGS["dense_decode"], 0.0572, PEAKS, "measured")
    pre = bench.dense_roofline(DENSE_CONFIGS["dense_prefill"], 1.62, PEAKS, "measured")
    assert dec["bound"] == "hbm" and dec["unit"] == "GB/s"
    assert pre["bound"] == "tensor" and pre["unit"] == "TFLOP/s"
    # e4m3 takes measured bf16 x 2
    assert pre["peak"] == pytest.approx(2 * PEAKS["bf16_tflops"])
    rec = json.load(open(RECORD))
    measured = rec["workloads"]["dense_decode"]["grouped_gemm_gate_up"]["traffic_bytes_per_launch"]
    assert abs(dec["algorithmic_bytes"] - measured) / measured < 0.02
    # achieved = bytes / time, frac = achieved / peak
    assert dec["achieved"] == pytest.approx(dec["algorithmic_bytes"] / 0.0572e-3 / 1e9, rel=1e-3)
    assert dec["frac"] == pytest.approx(dec["achieved"] / PEAKS["hbm_gbs"], rel=1e-3)


def test_traffic_record_used_only_where_it_applies():
    """The record's value, or None once the kernel sources differ from the
    ones it was taken on; None for workloads and kernels it does not hold."""
    import hashlib
    rec = json.load(open(RECORD))
    h = hashlib.sha256()
    for p in rec["sources"]:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    got = bench.kernel_traffic("grouped_gemm_gate_up", "decode")
    if h.hexdigest() == rec["source_sha256"]:
        assert got == rec["workloads"]["decode"]["grouped_gemm_gate_up"]["traffic_bytes_per_launch"]
    else:
        assert got is None
    assert "bf16" not in rec["workloads"]
    assert bench.kernel_traffic("grouped_gemm_gate_up", "bf16") is None
    assert bench.kernel_traffic("no_such_kernel", "decode") is None


def test_reference_arm_reports_the_same_config():
    """Both arms name the workload with the same `config` (the driver compares
    them); the reference arm runs the oracle on a bounded sample."""
    import argparse
    args = argparse.Namespace(steps=1, warmup=3, workload="tiny", ref_tokens=1, seed=0,
                              prenorm=False)
    res, cfg = bench.run_reference(args, 1, 0, 0)
    assert res["config"] == bench.moe_config(CONFIGS["tiny"], CONFIGS["tiny"].T, 1, False)
    assert res["impl"] == "reference" and res["metric"] == bench.METRIC
    assert res["e2e"]["value"] == res["value"] and res["cpu_baseline"]["value"] == res["value"]
