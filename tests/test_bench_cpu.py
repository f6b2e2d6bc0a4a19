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
    """Decode: 155 routed experts were touched plus the shared one; ncu read
    the gate/up GEMM's weights once, so the two counts agree within 0.5 %."""
    rec = json.load(open(RECORD))
    measured = rec["workloads"]["decode"]["grouped_gemm_gate_up"]["traffic_bytes_per_launch"]
    alg = bench.algorithmic_bytes_gemm1(CONFIGS["decode"], touched=156)
    assert abs(alg - measured) / measured < 0.005


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
    assert bench.kernel_traffic("grouped_gemm_gate_up", "skew") is None
    assert bench.kernel_traffic("no_such_kernel", "decode") is None
