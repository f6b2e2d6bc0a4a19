"""Benchmark of the MoE-layer forward (DeepSeek-V3 dims) on B200.

One step = one forward pass of the whole layer (router, permutation,
quantise-and-scatter, grouped gate/up GEMM + SwiGLU, grouped down GEMM,
combine) over one batch of synthetic tokens.  Default workload: the largest
single-GPU batch, skewed routing (T=16384 tokens, d_model 7168, 256 routed
experts top-8 + 1 shared, d_expert 2048, e4m3 blockwise weights and
activations with fp32 scales, bf16 I/O, router bias Zipf-ranked so that the
hottest expert carries about 10x the mean load).  --workload decode gives the
T=64 decode batch, whose gate/up GEMM is bound by HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill|skew|bf16|...|dense_decode|dense_prefill]

N > 1 (launched by torch.distributed.run) runs N independent replicas, one
per GPU (the layer has no exchange step on one node's replicas): value =
tokens of all ranks / max-over-ranks time.  Rank 0 prints one JSON line.
--impl reference times the oracle (plain CPU implementation) on the host
cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import (CONFIGS, DENSE_CONFIGS, make_dense_inputs, make_inputs,  # noqa: E402
                        make_residual)

METRIC = "MoE-layer tokens/s at DeepSeek-V3 dims"
DENSE_METRIC = "dense FFN-layer tokens/s at DeepSeek-V3 dims (first layers, d_ff 18432)"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return PEAKS_FALLBACK, "fallback"


def kernel_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record in
    profiles/roofline_traffic.json, or None when that record was taken on
    another workload or on a different version of the kernel sources."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "roofline_traffic.json")) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for pth in rec["sources"]:
            with open(os.path.join(ROOT, pth), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return float(rec["workloads"][workload][kernel]["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def dist_setup(n_gpus, backend: str | None = None):
    """One process per GPU (torch.distributed.run sets RANK/WORLD_SIZE/
    LOCAL_RANK/MASTER_*).  The replicas exchange nothing on the data path;
    the process group only carries the barrier and the max-over-ranks time."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank time over all ranks (the job finishes with its slowest rank)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step_max * 1e-3)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML in a
    background thread every ~2 ms while the timed region runs."""
    # NVML clocks-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []
        self.max_mhz = None
        self.err = None
        self._stop = None

    def _handle(self, nv):
        props = torch.cuda.get_device_properties(self.dev)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return nv.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
            except Exception:
                pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = int(vis.split(",")[self.dev]) if vis and vis.split(",")[0].isdigit() else self.dev
        return nv.nvmlDeviceGetHandleByIndex(idx)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception as e:  # no NVML: report it, do not fail the run
            self.err = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                         int(get_reasons(h))))
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(0.002)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *a):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": [self.err or "no samples"], "samples": 0}
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples), "source": "nvml"}


# --------------------------------------------------------------- our arm ---

def algorithmic_bytes_gemm1(cfg, touched: int) -> float:
    """Bytes the gate/up GEMM must move once: the weights of every touched
    expert (and the shared one), their scales, the permuted activations and
    scales in, H and its scales out."""
    d, de, Rs = cfg.d_model, cfg.d_expert, cfg.R_s
    es = 2 if cfg.precision == "bf16" else 1
    w = touched * (2 * de * d * es + (4 * (2 * de // 128) * (d // 128) if es == 1 else 0))
    a = Rs * d * es + (Rs * (d // 128) * 4 if es == 1 else 0)
    h = Rs * de * es + (Rs * (de // 128) * 4 if es == 1 else 0)
    return float(w + a + h)


def gemm1_flops(cfg) -> float:
    """FLOPs of the gate/up GEMM: 2 * R_s rows * 2 d_expert outputs * d_model."""
    return 2.0 * cfg.R_s * 2 * cfg.d_expert * cfg.d_model


def tensor_peak(cfg, peaks) -> float:
    """Dense tensor-core peak (TFLOP/s) of the GEMMs' operand type: measured
    bf16 GEMM throughput, times the nominal e4m3 / bf16 ratio (4.5 / 2.25)
    for the e4m3 precisions."""
    return peaks["bf16_tflops"] * (1 if cfg.precision == "bf16" else 2)


def moe_roofline(cfg, touched: int, ms: float, peaks, peak_kind: str):
    """Roofline of the gate/up GEMM (the dominant kernel): its algorithmic
    bytes (algorithmic_bytes_gemm1) and FLOPs (gemm1_flops); the bound is the
    roof with the longer floor at the measured peaks (HBM copy bandwidth, or
    the tensor peak of the operand type)."""
    nbytes = algorithmic_bytes_gemm1(cfg, touched)
    flops = gemm1_flops(cfg)
    tc = tensor_peak(cfg, peaks)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (tc * 1e12)
    src = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback"
    common = {"kernel": "grouped_gemm_gate_up", "algorithmic_bytes": nbytes,
              "algorithmic_flops": flops, "kernel_ms": round(ms, 4),
              "floor_ms": {"hbm": round(t_hbm * 1e3, 4), "tensor": round(t_tc * 1e3, 4)}}
    if t_tc > t_hbm:
        ach = flops / (ms * 1e-3) / 1e12
        sus = peaks.get("bf16_tflops_sustained")
        r = {"bound": "tensor", "achieved": round(ach, 1), "peak": tc, "unit": "TFLOP/s",
             "frac": round(ach / tc, 4),
             "peak_source": src + (" bf16_tflops x 2 (e4m3/bf16 nominal ratio)"
                                   if cfg.precision != "bf16" else " bf16_tflops")}
        if sus:
            tcs = sus * (1 if cfg.precision == "bf16" else 2)
            r["frac_of_sustained"] = round(ach / tcs, 4)
        return {**common, **r}
    ach = nbytes / (ms * 1e-3) / 1e9
    return {**common, "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
            "peak_source": src + " hbm_gbs"}


def layer_floor(cfg, touched: int, ms_step: float, peaks):
    """Floor of the whole layer: the longer of its HBM floor (every touched
    expert's weights and scales read once, x read and out written once) and
    its tensor floor (the two grouped GEMMs' FLOPs at the tensor peak); the
    router's binary32 logits run on the CUDA cores and are not counted in
    either.  frac = floor / measured step time."""
    d, de = cfg.d_model, cfg.d_expert
    es = 2 if cfg.precision == "bf16" else 1
    sc = 0 if es == 2 else 4 * ((2 * de // 128) * (d // 128) + (d // 128) * (de // 128))
    w = touched * (3 * de * d * es + sc)
    io = cfg.T * d * 2 * 2
    flops = 2.0 * cfg.R_s * 3 * de * d
    t_hbm = (w + io) / (peaks["hbm_gbs"] * 1e9) * 1e3
    t_tc = flops / (tensor_peak(cfg, peaks) * 1e12) * 1e3
    floor = max(t_hbm, t_tc)
    return {"bound": "tensor" if t_tc > t_hbm else "hbm", "floor_ms": round(floor, 4),
            "hbm_floor_ms": round(t_hbm, 4), "tensor_floor_ms": round(t_tc, 4),
            "frac": round(floor / ms_step, 4)}


def e2e_host_loop(call, x, d_model, steps, world, dev):
    """End-to-end steps through the public API with pinned host buffers: each
    step copies its x host -> device, runs the layer and copies out device ->
    host.  Two forms, both timed with CUDA events and max over ranks:
    serial (copy, layer, copy on one stream) and pipelined (the copies on a
    second stream, double-buffered, so step i+1's input and step i-1's
    result move while step i computes: the loop of a server).  -> ms per step
    (serial, pipelined)."""
    T = x.shape[0]
    stream = torch.cuda.current_stream()
    x_host = x.cpu().pin_memory()
    out_host = [torch.empty(T, d_model, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    out_dev = [torch.empty(T, d_model, dtype=torch.bfloat16, device=x.device) for _ in range(2)]

    def serial(n):
        for _ in range(n):
            x_dev[0].copy_(x_host, non_blocking=True)
            call(x_dev[0], out_dev[0])
            out_host[0].copy_(out_dev[0], non_blocking=True)

    copy = torch.cuda.Stream(device=x.device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]

    def pipelined(n, start):
        copy.wait_event(start)
        with torch.cuda.stream(copy):
            x_dev[0].copy_(x_host, non_blocking=True)
            ev_in[0].record(copy)
        for i in range(n):
            b = i & 1
            stream.wait_event(ev_in[b])
            call(x_dev[b], out_dev[b])
            ev_done[b].record(stream)
            with torch.cuda.stream(copy):
                if i + 1 < n:
                    if i >= 1:
                        copy.wait_event(ev_done[b ^ 1])  # step i-1 has read this buffer
                    x_dev[b ^ 1].copy_(x_host, non_blocking=True)
                    ev_in[b ^ 1].record(copy)
                copy.wait_event(ev_done[b])
                out_host[b].copy_(out_dev[b], non_blocking=True)

    times = []
    for form in ("serial", "pipelined"):
        warm = torch.cuda.Event()
        warm.record(stream)
        serial(2) if form == "serial" else pipelined(2, warm)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if form == "serial":
            serial(steps)
            e1.record(stream)
        else:
            pipelined(steps, e0)
            stream.wait_stream(copy)
            e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        times.append(max_over_ranks(e0.elapsed_time(e1), world, dev) / steps)
    return times[0], times[1]


def moe_config(cfg, T: int, world: int, prenorm: bool) -> dict:
    """The line's `config`: the workload only, identical in both arms."""
    return {
        "workload": ("pre-norm block (h + MoE(RMSNorm(h)), fused) " if prenorm else "")
                    + f"{cfg.name}: T={T}, d_model={cfg.d_model}, {cfg.n_experts} experts "
                    f"top-{cfg.top_k} + {cfg.n_shared} shared, d_expert={cfg.d_expert}, "
                    + ({"fp8": "e4m3 1x128/128x128 blockwise, fp32 scales, bf16 I/O",
                        "fp8_ue8m0": "e4m3 1x128/128x128 blockwise, power-of-two (UE8M0) "
                                     "scales, bf16 I/O"}.get(cfg.precision, "bf16")),
        "tokens_per_gpu": T,
        "parallelism": "replicas" if world > 1 else "single GPU",
        "l2": "inputs larger than L2: the touched experts' weights (GB per step) stream through "
              "every step",
    }


def dense_config(cfg, T: int, world: int, prenorm: bool) -> dict:
    """The dense line's `config`, identical in both arms."""
    return {
        "workload": ("pre-norm block (h + FFN(RMSNorm(h)), fused) " if prenorm else "")
                    + f"{cfg.name}: T={T}, d_model={cfg.d_model}, d_ff={cfg.d_ff}, "
                    + {"fp8": "e4m3 1x128/128x128 blockwise, fp32 scales, bf16 I/O",
                       "fp8_ue8m0": "e4m3 blockwise, power-of-two scales, bf16 I/O"}.get(
                           cfg.precision, "bf16"),
        "tokens_per_gpu": T,
        "parallelism": "replicas" if world > 1 else "single GPU",
        "l2": f"inputs larger than L2: {3 * cfg.d_model * cfg.d_ff / 1e6:.0f} MB of weights "
              "stream through every step",
    }


def run_ours(args, world, rank, local):
    import sparse_moe_transformer_fwd_b200 as moe
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = CONFIGS[args.workload]
    inp = make_inputs(cfg, seed=args.seed + rank, device=dev)
    layer = moe.MoELayer(inp["w_router"], inp["bias"], inp["w13"], inp["w2"], top_k=cfg.top_k,
                         n_shared=cfg.n_shared, precision=cfg.precision)
    del inp["w13"], inp["w2"]
    torch.cuda.empty_cache()
    T = cfg.T
    if args.prenorm:
        # the FFN block: residual stream h in, pre-norm fused, h + MoE(x) out
        x, gamma = make_residual(cfg, seed=args.seed + rank, device=dev)
        call = lambda xx, out, topk_idx_out=None: layer.forward_prenorm(
            xx, gamma, 1e-6, out=out, topk_idx_out=topk_idx_out)
    else:
        x = inp["x"]
        call = layer
    out = torch.empty(T, cfg.d_model, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(T, cfg.top_k, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        call(x, out=out, topk_idx_out=idx)
    torch.cuda.synchronize()
    status = layer.check_status(T)
    if status != 0:
        raise RuntimeError(f"device status {status}: {moe.moe_last_error()}")
    n_launch = moe.moe_last_launch_count()
    names = moe.moe_last_launch_names()  # the library's own record of its launches
    touched = int(torch.unique(idx).numel()) + cfg.n_shared
    counts = torch.bincount(idx.reshape(-1).long(), minlength=cfg.n_experts)

    # ---- device-timed region: K steps, inputs resident in HBM, nothing but the
    # layer's own launches between the two events
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for k in range(args.steps):
            call(x, out=out, topk_idx_out=idx)
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_total = max_over_ranks(start.elapsed_time(stop), world, dev)
    ms_step = ms_total / args.steps

    # ---- the dominant kernel (gate/up GEMM), bracketed by CUDA events on
    # every step of a separate pass of K steps (an event between two launches
    # stops their programmatic overlap, so this pass is not the timed one)
    gi = names.index("grouped_gemm_gate_up")
    g_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for k in range(args.steps):
        moe.moe_set_kernel_events([None] * gi + list(g_ev[k]))
        call(x, out=out, topk_idx_out=idx)
    moe.moe_set_kernel_events(None)
    torch.cuda.synchronize()
    g1_ms = float(np.mean([a.elapsed_time(b) for a, b in g_ev]))

    # ---- per-kernel breakdown (separate pass, every launch bracketed)
    nb = min(args.steps, 10)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_launch + 1)] for _ in range(nb)]
    for k in range(nb):
        moe.moe_set_kernel_events(ev[k])
        call(x, out=out, topk_idx_out=idx)
    moe.moe_set_kernel_events(None)
    torch.cuda.synchronize()
    kmean = np.array([[ev[k][i].elapsed_time(ev[k][i + 1]) for i in range(n_launch)]
                      for k in range(nb)]).mean(0)

    # ---- end to end through the public API with host buffers
    ms_serial, ms_e2e = e2e_host_loop(lambda xx, oo: call(xx, out=oo), x, cfg.d_model,
                                      args.steps, world, dev)
    status = layer.check_status(T)
    if status != 0:
        raise RuntimeError(f"device status {status}: {moe.moe_last_error()}")

    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    g1_bytes = algorithmic_bytes_gemm1(cfg, touched)
    tokens_total = T * world
    value = job_throughput(T, world, ms_step)
    res = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.precision == "bf16" else "e4m3",
        "data": "synthetic (seeded; random-init weights of the DeepSeek-V3 MoE layer shape)",
        "config": moe_config(cfg, T, world, args.prenorm),
        "routing": {"touched_experts": touched,
                    "gate_up_algorithmic_bytes": int(g1_bytes),
                    "expert_load_max_over_mean": round(float(counts.max()) / (T * cfg.top_k / cfg.n_experts), 2),
                    "experts_empty": int((counts == 0).sum())},
        "roofline": {**moe_roofline(cfg, touched, g1_ms, peaks, peak_kind),
                     "kernel_ms_from": "CUDA events around this kernel on every step of a "
                                       "separate pass of K steps",
                     "traffic": kernel_traffic("grouped_gemm_gate_up", cfg.name),
                     "traffic_source": "profiles/roofline_traffic.json (ncu "
                                       "dram__bytes_read+write per launch)"},
        "layer_roofline": layer_floor(cfg, touched, ms_step, peaks),
        "kernels_ms": {n: round(float(v), 4) for n, v in zip(names, kmean)},
        "kernels_ms_note": "per-kernel means from a separate pass of the same call with every "
                           "launch bracketed by CUDA events",
        "e2e": {"value": round(tokens_total / (ms_e2e * 1e-3), 1), "unit": "tokens/s",
                "ms_per_step": round(ms_e2e, 4),
                "h2d_bytes_per_step": int(x.numel() * x.element_size()),
                "d2h_bytes_per_step": int(out.numel() * out.element_size()),
                "form": "pinned host x in, out back every step; copies on a second stream, "
                        "double-buffered, overlapping the neighbouring steps' compute",
                "serial": {"value": round(tokens_total / (ms_serial * 1e-3), 1),
                           "ms_per_step": round(ms_serial, 4),
                           "form": "copy in, layer, copy out on one stream"}},
        "gpu_launches": n_launch * args.steps,
        "clocks": clk.summary(),
    }
    return res, cfg


# ------------------------------------------------------ dense layer arm ---

def dense_roofline(cfg, ms: float, peaks, peak_kind: str):
    """Roofline of the dense gate/up GEMM: its algorithmic bytes (weights,
    their scales, x codes and scales in, H codes and scales out) and FLOPs;
    the bound is the roof with the longer floor at the measured peaks (HBM
    copy bandwidth; tensor: measured bf16 GEMM x 2 for e4m3, the nominal
    4.5 / 2.25 ratio)."""
    T, d, f = cfg.T, cfg.d_model, cfg.d_ff
    es = 2 if cfg.precision == "bf16" else 1
    sc = 0 if es == 2 else 4
    nbytes = (2 * f * d * es + sc * (2 * f // 128) * (d // 128) + T * d * es + sc * T * (d // 128)
              + T * f * es + sc * T * (f // 128))
    flops = 2.0 * T * d * 2 * f
    tc_peak = peaks["bf16_tflops"] * (1 if es == 2 else 2)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    src = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback"
    if t_tc > t_hbm:
        ach = flops / (ms * 1e-3) / 1e12
        return {"kernel": "grouped_gemm_gate_up", "bound": "tensor", "achieved": round(ach, 1),
                "peak": tc_peak, "unit": "TFLOP/s", "frac": round(ach / tc_peak, 4),
                "peak_source": src + (" bf16_tflops x 2 (e4m3)" if es == 1 else " bf16_tflops"),
                "algorithmic_flops": flops, "kernel_ms": round(ms, 4), "traffic": None}
    ach = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "grouped_gemm_gate_up", "bound": "hbm", "achieved": round(ach, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
            "peak_source": src + " hbm_gbs", "algorithmic_bytes": nbytes,
            "kernel_ms": round(ms, 4), "traffic": kernel_traffic("grouped_gemm_gate_up", cfg.name)}


def run_dense(args, world, rank, local):
    import sparse_moe_transformer_fwd_b200 as moe
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = DENSE_CONFIGS[args.workload]
    inp = make_dense_inputs(cfg, seed=args.seed + rank, device=dev)
    layer = moe.DenseFFN(inp["w13"], inp["w2"], precision=cfg.precision)
    del inp["w13"], inp["w2"]
    torch.cuda.empty_cache()
    T = cfg.T
    if args.prenorm:
        x, gamma = make_residual(cfg, seed=args.seed + rank, device=dev)
        call = lambda xx, out: layer.forward_prenorm(xx, gamma, 1e-6, out=out)
    else:
        x = inp["x"]
        call = lambda xx, out: layer(xx, out=out)
    out = torch.empty(T, cfg.d_model, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        call(x, out)
    torch.cuda.synchronize()
    if layer.check_status(T) != 0:
        raise RuntimeError(f"device status: {moe.moe_last_error()}")
    n_launch = moe.moe_last_launch_count()
    names = moe.moe_last_launch_names()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for k in range(args.steps):
            call(x, out)
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_step = max_over_ranks(start.elapsed_time(stop), world, dev) / args.steps
    # the gate/up GEMM bracketed on every step of a separate pass
    gi = names.index("grouped_gemm_gate_up")
    g_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for k in range(args.steps):
        moe.moe_set_kernel_events([None] * gi + list(g_ev[k]))
        call(x, out)
    moe.moe_set_kernel_events(None)
    torch.cuda.synchronize()
    g1_ms = float(np.mean([a.elapsed_time(b) for a, b in g_ev]))
    nb = min(args.steps, 10)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_launch + 1)] for _ in range(nb)]
    for k in range(nb):
        moe.moe_set_kernel_events(ev[k])
        call(x, out)
    moe.moe_set_kernel_events(None)
    torch.cuda.synchronize()
    kmean = np.array([[ev[k][i].elapsed_time(ev[k][i + 1]) for i in range(n_launch)]
                      for k in range(nb)]).mean(0)
    # end to end with host buffers
    ms_serial, ms_e2e = e2e_host_loop(call, x, cfg.d_model, args.steps, world, dev)
    if layer.check_status(T) != 0:
        raise RuntimeError(f"device status: {moe.moe_last_error()}")
    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    res = {
        "metric": DENSE_METRIC, "value": round(job_throughput(T, world, ms_step), 1),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.precision == "bf16" else "e4m3",
        "data": "synthetic (seeded; random-init weights of the DeepSeek-V3 dense FFN shape)",
        "config": dense_config(cfg, T, world, args.prenorm),
        "roofline": dense_roofline(cfg, g1_ms, peaks, peak_kind),
        "kernels_ms": {n: round(float(v), 4) for n, v in zip(names, kmean)},
        "e2e": {"value": round(T * world / (ms_e2e * 1e-3), 1), "unit": "tokens/s",
                "ms_per_step": round(ms_e2e, 4),
                "h2d_bytes_per_step": int(x.numel() * x.element_size()),
                "d2h_bytes_per_step": int(out.numel() * out.element_size()),
                "form": "pinned host x in, out back every step; copies on a second stream, "
                        "double-buffered, overlapping the neighbouring steps' compute",
                "serial": {"value": round(T * world / (ms_serial * 1e-3), 1),
                           "ms_per_step": round(ms_serial, 4)}},
        "gpu_launches": n_launch * args.steps,
        "clocks": clk.summary(),
    }
    return res, cfg


def dense_oracle_time(cfg, n_tokens: int, seed: int, reps: int = 1):
    """Time the oracle's dense layer on n_tokens rows of the batch (rows are
    independent; the weights' quantisation is part of every call)."""
    import oracle
    from threadpoolctl import threadpool_limits
    inp = make_dense_inputs(cfg, seed=seed)
    u16 = lambda t: t.detach().contiguous().view(torch.int16).numpy().view(np.uint16)
    tokens = list(range(0, cfg.T, max(1, cfg.T // n_tokens)))[:n_tokens]
    x, w13, w2 = u16(inp["x"][tokens]), u16(inp["w13"]), u16(inp["w2"])
    del inp
    times = []
    with threadpool_limits(limits=1):
        for _ in range(reps):
            t0 = time.perf_counter()
            oracle.dense_ffn(x, w13, w2, precision=cfg.precision)
            times.append(time.perf_counter() - t0)
    return times, len(tokens)


# ----------------------------------------------------- oracle (CPU) arm ---

def oracle_sample_time(cfg, dev, n_tokens: int, seed: int, reps: int = 1):
    """Time the oracle's whole layer on a sample of n_tokens of the workload's
    batch (tokens are independent), BLAS limited to one thread."""
    import oracle
    from threadpoolctl import threadpool_limits
    inp = make_inputs(cfg, seed=seed, device=dev)
    u16 = lambda t: t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    tokens = list(range(0, cfg.T, max(1, cfg.T // n_tokens)))[:n_tokens]
    x = u16(inp["x"][tokens])
    wr = u16(inp["w_router"])
    b = inp["bias"].cpu().numpy()
    # host copies of the experts the sample touches (inputs, copied before timing)
    import oracle as _o
    sel = set()
    idx, _, _ = _o.route(_o.router_logits(x, wr), b, cfg.top_k)
    sel.update(int(e) for e in idx.reshape(-1))
    sel.add(cfg.n_experts)
    experts = {e: (u16(inp["w13"][e]), u16(inp["w2"][e])) for e in sorted(sel)}
    del inp
    times = []
    with threadpool_limits(limits=1):
        for _ in range(reps):
            t0 = time.perf_counter()
            oracle.moe_layer(x, wr, b, lambda e: experts[e], n_experts=cfg.n_experts,
                             top_k=cfg.top_k, n_shared=cfg.n_shared, precision=cfg.precision)
            times.append(time.perf_counter() - t0)
    return times, len(tokens), len(sel)


def oracle_sample_time_all_cores(cfg, dev, per_worker: int, seed: int):
    """The oracle's whole layer on all host cores: one thread per core, each
    running the oracle (single-threaded per op, BLAS held to one thread) on
    its own chunk of per_worker tokens of the batch (tokens are independent;
    the C core and numpy release the interpreter lock).  The workers share
    the host copies of the experts the sample touches, made before timing.
    The worker count is the number of usable cores, lowered only if host
    memory cannot hold the copies plus ~1 GB of temporaries per worker.
    -> (wall seconds, tokens, workers, experts touched)."""
    import concurrent.futures as cf

    import psutil
    from threadpoolctl import threadpool_limits

    import oracle
    cores = len(os.sched_getaffinity(0))
    inp = make_inputs(cfg, seed=seed, device=dev)
    u16 = lambda t: t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    wr = u16(inp["w_router"])
    b = inp["bias"].cpu().numpy()
    expert_bytes = 3 * cfg.d_expert * cfg.d_model * 2
    avail = psutil.virtual_memory().available
    workers = cores
    while workers > 1:
        n_tok = workers * per_worker
        stride = max(1, cfg.T // n_tok)
        tokens = list(range(0, cfg.T, stride))[:n_tok]
        x_all = u16(inp["x"][tokens])
        idx, _, _ = oracle.route(oracle.router_logits(x_all, wr), b, cfg.top_k)
        sel = sorted(set(int(e) for e in idx.reshape(-1)) | {cfg.n_experts})
        if len(sel) * expert_bytes + workers * (1 << 30) + (8 << 30) <= avail:
            break
        workers //= 2
    if workers <= 1:
        return None
    experts = {e: (u16(inp["w13"][e]), u16(inp["w2"][e])) for e in sel}
    del inp
    chunks = [x_all[i * per_worker:(i + 1) * per_worker] for i in range(workers)]

    def one(xc):
        return oracle.moe_layer(xc, wr, b, lambda e: experts[e], n_experts=cfg.n_experts,
                                top_k=cfg.top_k, n_shared=cfg.n_shared,
                                precision=cfg.precision)["out"].shape[0]

    with threadpool_limits(limits=1), cf.ThreadPoolExecutor(workers) as ex:
        t0 = time.perf_counter()
        done = sum(ex.map(one, chunks))
        wall = time.perf_counter() - t0
    return wall, done, workers, len(sel)


def cpu_baseline_ours(cfg, dev, args):
    """cpu_baseline of the default arm: the oracle on all host cores (one
    thread per core over token chunks), with the single-threaded form beside it."""
    times, ntok, nexp = oracle_sample_time(cfg, dev, args.cpu_baseline_tokens, args.seed)
    single = {"value": round(ntok / times[0], 4), "unit": "tokens/s", "cores": 1,
              "sample": f"{ntok} tokens of the {cfg.name} batch through the oracle's whole "
                        f"layer ({nexp} experts incl. their weight quantisation), "
                        f"{times[0]:.1f} s, 1 thread"}
    par = oracle_sample_time_all_cores(cfg, dev, args.cpu_baseline_tokens, args.seed)
    base = {"kind": "oracle", "cpu": cpu_model(), "single_thread": single}
    if par is None:
        return {**single, **base, "all_cores": "not run: host memory too small"}
    wall, ntok_p, workers, nexp_p = par
    return {"value": round(ntok_p / wall, 4), "unit": "tokens/s", "cores": workers, **base,
            "sample": f"{ntok_p} tokens of the {cfg.name} batch, {args.cpu_baseline_tokens} per "
                      f"thread on {workers} threads (one per core), each through the oracle's "
                      f"whole layer ({nexp_p} experts touched, each thread quantising the "
                      f"weights of its own experts), {wall:.1f} s wall"}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for l in f:
                if l.startswith("model name"):
                    return l.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference_dense(args, world):
    cfg = DENSE_CONFIGS[args.workload]
    dense_oracle_time(cfg, args.ref_tokens, args.seed, reps=1)
    times, ntok = dense_oracle_time(cfg, args.ref_tokens, args.seed, reps=args.steps)
    s_step = statistics.mean(times)
    value = ntok / s_step
    sample = (f"{ntok} tokens of the {cfg.name} batch per step through the oracle's dense layer "
              "(weight quantisation, binary64 GEMMs); C core and numpy on 1 thread")
    return {
        "metric": DENSE_METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(s_step * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": dense_config(cfg, cfg.T, world, args.prenorm),
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "cpu": cpu_model()},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }, cfg


def run_reference(args, world, rank, local):
    if rank != 0:
        return None
    if args.workload in DENSE_CONFIGS:
        return run_reference_dense(args, world)
    cfg = CONFIGS[args.workload]
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    n_tok = args.ref_tokens
    step_times = []
    warm, _, _ = oracle_sample_time(cfg, dev, n_tok, args.seed, reps=max(1, min(args.warmup, 1)))
    times, ntok, nexp = oracle_sample_time(cfg, dev, n_tok, args.seed, reps=args.steps)
    step_times = times
    s_step = statistics.mean(step_times)
    value = ntok / s_step
    sample = (f"{ntok} tokens of the {cfg.name} batch per step through the oracle's whole layer "
              f"(routing, permutation, quantisation incl. the {nexp} touched experts' weights, "
              f"binary64 expert GEMMs, combine); C core and numpy on 1 thread")
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(s_step * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": moe_config(cfg, cfg.T, world, args.prenorm),
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "cpu": cpu_model()},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }, cfg


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(CONFIGS) + list(DENSE_CONFIGS), default="skew")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ref-tokens", type=int, default=1,
                    help="tokens of the batch per oracle step (reference arm)")
    ap.add_argument("--cpu-baseline-tokens", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prenorm", action="store_true",
                    help="time the FFN block with its fused pre-norm and residual")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            r = run_reference(args, world, rank, local)
            if r is not None:
                print(json.dumps(r[0]), flush=True)
            return
        dense = args.workload in DENSE_CONFIGS
        r = (run_dense if dense else run_ours)(args, world, rank, local)
        if r is not None:
            res, cfg = r
            if world == 1 and not args.no_cpu_baseline and dense:
                times, ntok = dense_oracle_time(cfg, args.cpu_baseline_tokens, args.seed)
                res["cpu_baseline"] = {
                    "value": round(ntok / times[0], 4), "unit": "tokens/s", "cores": 1,
                    "kind": "oracle",
                    "sample": f"{ntok} tokens of the {cfg.name} batch through the oracle's dense "
                              f"layer (incl. its weight quantisation), {times[0]:.1f} s, 1 thread",
                    "cpu": cpu_model()}
            elif world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline_ours(cfg, torch.device("cuda", local), args)
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
