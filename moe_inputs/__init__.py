"""Seeded synthetic workloads for the DeepSeek-V3/R1 MoE FFN layer.

This module is the only code that both the oracle-side tests and the CUDA
path's callers share.  It holds workload shapes and random-value recipes and
nothing of the layer's arithmetic (no routing, quantisation, GEMM or combine).

Shapes follow the architecture card of "DeepSeek-R1" on
llm-architectures-explained.vercel.app ("Every architecture field" table:
d_model 7168, 256 routed experts, 8 active, d_expert 2048, 1 shared expert of
width 2048).  The value distributions are the workload recipes of this
project (x ~ N(0,1) RMS-normalised; expert weights N(0, sigma); router bias
uniform, zero, or Zipf-ranked), since the pages print no activations or
weights.

Every tensor is drawn from its own torch generator, seeded by a fixed mix of
(seed, tensor id, expert index), so any single expert can be regenerated on
its own on the same device type.  CPU and CUDA generators give different
streams: a test that compares two computations must feed both the same
materialised tensors.
"""
from __future__ import annotations

import dataclasses
import json
import math
import os

import torch

__all__ = ["MoEConfig", "CONFIGS", "make_inputs", "expert_weights", "skew_bias_scale",
           "make_residual", "DenseConfig", "DENSE_CONFIGS", "make_dense_inputs"]

_HERE = os.path.dirname(os.path.abspath(__file__))

# tensor ids for seeding
_TID_X, _TID_WR, _TID_BIAS, _TID_W13, _TID_W2, _TID_RANK, _TID_H, _TID_G = 1, 2, 3, 4, 5, 6, 7, 8
_TID_DW13, _TID_DW2 = 9, 10


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int              # tokens
    d_model: int
    n_experts: int      # routed experts E
    top_k: int
    d_expert: int
    n_shared: int       # 0 or 1 shared experts (width d_expert)
    precision: str      # "bf16", "fp8" (FP32 block scales) or "fp8_ue8m0" (power-of-two scales)
    w_std: float        # std of expert weights
    wr_std: float       # std of router weights
    bias: str           # "uniform" (U(-0.1, 0.1)), "zero", or "zipf"
    routed_scale: float = 1.0

    @property
    def R(self) -> int:           # routed rows
        return self.T * self.top_k

    @property
    def R_s(self) -> int:         # routed rows + shared rows
        return self.T * self.top_k + self.T * self.n_shared

    def with_(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    def flops_per_token(self) -> float:
        """Algorithmic FLOPs per token: router plus (k + shared) gated experts."""
        d, de = self.d_model, self.d_expert
        expert = 2.0 * 3 * d * de
        router = 2.0 * d * self.n_experts
        return (self.top_k + self.n_shared) * expert + router


_DS = dict(d_model=7168, n_experts=256, top_k=8, d_expert=2048, n_shared=1,
           w_std=0.006, wr_std=0.006)

CONFIGS = {
    "tiny": MoEConfig("tiny", T=128, d_model=512, n_experts=16, top_k=4, d_expert=256,
                      n_shared=1, precision="bf16", w_std=0.02, wr_std=1.0 / math.sqrt(512),
                      bias="uniform"),
    "decode": MoEConfig("decode", T=64, precision="fp8", bias="uniform", **_DS),
    "prefill": MoEConfig("prefill", T=4096, precision="fp8", bias="zero", **_DS),
    "skew": MoEConfig("skew", T=16384, precision="fp8", bias="zipf", **_DS),
    "bf16": MoEConfig("bf16", T=8192, precision="bf16", bias="zero", **_DS),
    # the decode and prefill batches with the UE8M0 (power-of-two) block scales
    "decode_ue8m0": MoEConfig("decode_ue8m0", T=64, precision="fp8_ue8m0", bias="uniform", **_DS),
    "prefill_ue8m0": MoEConfig("prefill_ue8m0", T=4096, precision="fp8_ue8m0", bias="zero", **_DS),
    # profiling-size stand-in for the decode batch: same per-expert shapes,
    # 32 routed experts, so every buffer is a few GB at most
    "decode_small": MoEConfig("decode_small", T=64, precision="fp8", bias="uniform",
                              **{**_DS, "n_experts": 32}),
    # profiling-size stand-in for the large batches: ~1000 rows per expert
    "prefill_small": MoEConfig("prefill_small", T=4096, precision="fp8", bias="zero",
                               **{**_DS, "n_experts": 32}),
    "prefill_small_ue8m0": MoEConfig("prefill_small_ue8m0", T=4096, precision="fp8_ue8m0",
                                     bias="zero", **{**_DS, "n_experts": 32}),
    # profiling-size stand-in for the skew batch: the same Zipf-ranked bias
    # over 32 routed experts, so one expert carries several times the mean
    "skew_small": MoEConfig("skew_small", T=4096, precision="fp8", bias="zipf",
                            **{**_DS, "n_experts": 32}),
}


def _seed(seed: int, tid: int, expert: int = 0) -> int:
    # splitmix64-style mix of the three ids into one 63-bit seed
    z = (seed * 0x9E3779B97F4A7C15 + tid * 0xBF58476D1CE4E5B9 + (expert + 1) * 0x94D049BB133111EB)
    z &= (1 << 64) - 1
    z ^= z >> 31
    z = (z * 0xD6E8FEB86659FD93) & ((1 << 64) - 1)
    z ^= z >> 32
    return z & ((1 << 63) - 1)


def _gen(device, seed, tid, expert=0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, tid, expert))
    return g


def skew_bias_scale() -> float:
    """Scale c of the Zipf-ranked router bias, written by oracle/calibrate_skew.py."""
    path = os.path.join(_HERE, "skew_bias_scale.json")
    with open(path) as f:
        return float(json.load(f)["c"])


def zipf_bias(E: int, seed: int, c: float, s: float = 1.1) -> torch.Tensor:
    """b_e = c * (-s * ln r_e), r a seeded permutation of the ranks 1..E (fp32, CPU)."""
    g = _gen("cpu", seed, _TID_RANK)
    ranks = torch.randperm(E, generator=g).to(torch.float64) + 1.0
    return (c * (-s * torch.log(ranks))).to(torch.float32)


def make_x(cfg: MoEConfig, seed: int = 0, device="cpu", T: int | None = None) -> torch.Tensor:
    """x ~ N(0,1), each row divided by sqrt(mean(x^2) + 1e-6), rounded to bf16."""
    T = cfg.T if T is None else T
    x = torch.randn(T, cfg.d_model, generator=_gen(device, seed, _TID_X), device=device,
                    dtype=torch.float32)
    x = x / torch.sqrt((x * x).mean(dim=1, keepdim=True) + 1e-6)
    return x.to(torch.bfloat16)


def make_residual(cfg: MoEConfig, seed: int = 0, device="cpu", T: int | None = None):
    """Inputs of the pre-norm block: the residual stream h ~ N(0, 1) * s_t with
    a per-token scale s_t ~ exp(U(-1, 2)) (rows of very different norms), and
    the RMSNorm weight gamma ~ U(0.5, 1.5); both bf16."""
    T = cfg.T if T is None else T
    g = _gen(device, seed, _TID_H)
    h = torch.randn(T, cfg.d_model, generator=g, device=device, dtype=torch.float32)
    h = h * torch.exp(torch.rand(T, 1, generator=g, device=device) * 3.0 - 1.0)
    gamma = torch.rand(cfg.d_model, generator=_gen(device, seed, _TID_G), device=device) + 0.5
    return h.to(torch.bfloat16), gamma.to(torch.bfloat16)


def make_router(cfg: MoEConfig, seed: int = 0, device="cpu"):
    w = torch.randn(cfg.n_experts, cfg.d_model, generator=_gen(device, seed, _TID_WR),
                    device=device, dtype=torch.float32) * cfg.wr_std
    if cfg.bias == "uniform":
        b = (torch.rand(cfg.n_experts, generator=_gen(device, seed, _TID_BIAS), device=device,
                        dtype=torch.float32) * 0.2 - 0.1)
    elif cfg.bias == "zero":
        b = torch.zeros(cfg.n_experts, device=device, dtype=torch.float32)
    elif cfg.bias == "zipf":
        b = zipf_bias(cfg.n_experts, seed, skew_bias_scale()).to(device)
    else:
        raise ValueError(cfg.bias)
    return w.to(torch.bfloat16), b.contiguous()


def expert_weights(cfg: MoEConfig, e: int, seed: int = 0, device="cpu"):
    """(w13 [2*d_e, d] gate rows then up rows, w2 [d, d_e]) of expert e, bf16.

    e == n_experts is the shared expert."""
    d, de = cfg.d_model, cfg.d_expert
    w13 = torch.randn(2 * de, d, generator=_gen(device, seed, _TID_W13, e), device=device,
                      dtype=torch.float32) * cfg.w_std
    w2 = torch.randn(d, de, generator=_gen(device, seed, _TID_W2, e), device=device,
                     dtype=torch.float32) * cfg.w_std
    return w13.to(torch.bfloat16), w2.to(torch.bfloat16)


def make_inputs(cfg: MoEConfig, seed: int = 0, device="cpu", identical_experts: bool = False):
    """All layer inputs as torch tensors on `device`.

    Returns dict(x [T,d] bf16, w_router [E,d] bf16, bias [E] fp32,
    w13 [E+S, 2*d_e, d] bf16, w2 [E+S, d, d_e] bf16), S = n_shared; the shared
    expert is the last slot.  identical_experts=True gives every routed expert
    the weights of expert 0 (a special case used by the oracle's pins)."""
    x = make_x(cfg, seed, device)
    w_r, b = make_router(cfg, seed, device)
    n_slots = cfg.n_experts + cfg.n_shared
    d, de = cfg.d_model, cfg.d_expert
    w13 = torch.empty(n_slots, 2 * de, d, dtype=torch.bfloat16, device=device)
    w2 = torch.empty(n_slots, d, de, dtype=torch.bfloat16, device=device)
    for e in range(n_slots):
        src = 0 if (identical_experts and e < cfg.n_experts) else e
        a, c = expert_weights(cfg, src, seed, device)
        w13[e].copy_(a)
        w2[e].copy_(c)
    return dict(x=x, w_router=w_r, bias=b, w13=w13, w2=w2)


# ----------------------------------------------------------- dense layers --

@dataclasses.dataclass(frozen=True)
class DenseConfig:
    """A dense gated FFN layer: the card's first layers ("Every architecture
    field": layout 3 x dense then 58 x MoE; ffns.dense gated, d_ff 18432)."""
    name: str
    T: int
    d_model: int
    d_ff: int
    precision: str      # "bf16", "fp8" or "fp8_ue8m0", as for the MoE layer
    w_std: float

    def with_(self, **kw) -> "DenseConfig":
        return dataclasses.replace(self, **kw)

    def flops_per_token(self) -> float:
        return 2.0 * 3 * self.d_model * self.d_ff


DENSE_CONFIGS = {
    "dense_tiny": DenseConfig("dense_tiny", T=100, d_model=512, d_ff=768, precision="fp8",
                              w_std=0.02),
    # the MoE workloads' batches through a dense first layer (same value recipe)
    "dense_decode": DenseConfig("dense_decode", T=64, d_model=7168, d_ff=18432,
                                precision="fp8", w_std=0.006),
    "dense_prefill": DenseConfig("dense_prefill", T=4096, d_model=7168, d_ff=18432,
                                 precision="fp8", w_std=0.006),
}


def make_dense_inputs(cfg: DenseConfig, seed: int = 0, device="cpu"):
    """dict(x [T, d] bf16 (as make_x), w13 [2*d_ff, d] bf16 gate rows then up
    rows, w2 [d, d_ff] bf16), weights N(0, w_std)."""
    x = make_x(cfg, seed, device)
    d, f = cfg.d_model, cfg.d_ff
    w13 = torch.randn(2 * f, d, generator=_gen(device, seed, _TID_DW13), device=device,
                      dtype=torch.float32) * cfg.w_std
    w2 = torch.randn(d, f, generator=_gen(device, seed, _TID_DW2), device=device,
                     dtype=torch.float32) * cfg.w_std
    return dict(x=x, w13=w13.to(torch.bfloat16), w2=w2.to(torch.bfloat16))
