"""Calibrate the scale c of the Zipf-ranked router bias of the skewed-routing
workload (T=16384, DeepSeek-V3 dims): b_e = c * (-1.1 * ln r_e) with r a
seeded permutation of the ranks 1..256, c chosen by bisection so that the
hottest expert receives 10x the mean load (T*k/E) under the oracle's router.

The bias only steers selection (routing-only bias of "Local Balanced Routing
to Experts"); here it is used in reverse, to make an imbalanced workload.
A pure Zipf(1.1) popularity over 256 experts would put 256 / H(256, 1.1) = 53x
the mean on the hottest expert, above what top-8-of-256 allows (32x), so the
Zipf shape is kept for the ranks and the peak is set to 10x.

Runs on the CPU only (oracle router on CPU-generated inputs of the same
distribution; calibrating on T=4096 tokens of it).  Writes
moe_inputs/skew_bias_scale.json.
"""
from __future__ import annotations

import json
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from moe_inputs import CONFIGS, make_x, make_router, zipf_bias  # noqa: E402

TARGET = 10.0


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def main(T_cal: int = 4096, seed: int = 0):
    cfg = CONFIGS["skew"]
    E, k = cfg.n_experts, cfg.top_k
    t0 = time.time()
    x = make_x(cfg, seed, "cpu", T=T_cal)
    w_r, _ = make_router(cfg.with_(bias="zero"), seed, "cpu")
    logits = oracle.router_logits(_u16(x), _u16(w_r))
    print(f"logits {logits.shape} in {time.time() - t0:.1f}s", flush=True)

    def ratio(c):
        b = zipf_bias(E, seed, c).numpy()
        idx, _, _ = oracle.route(logits, b, k)
        load = np.bincount(idx.reshape(-1), minlength=E)
        return load.max() / (T_cal * k / E)

    lo, hi = 0.0, 1.0
    while ratio(hi) < TARGET:
        hi *= 2
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if ratio(mid) < TARGET:
            lo = mid
        else:
            hi = mid
    c = 0.5 * (lo + hi)
    r = ratio(c)
    out = dict(c=c, achieved_ratio=float(r), target_ratio=TARGET, T_calibration=T_cal,
               seed=seed, zipf_s=1.1,
               note="written by oracle/calibrate_skew.py from the oracle router")
    path = os.path.join(ROOT, "moe_inputs", "skew_bias_scale.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
