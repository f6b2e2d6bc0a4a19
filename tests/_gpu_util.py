"""Helpers shared by the GPU parity tests: tensor conversions, running the
CUDA path through the C ABI, running the oracle on the same inputs, and the
output tolerance (relative L2 <= 1e-3 and max |diff| <= 1e-2 * RMS of the
oracle output)."""
from __future__ import annotations

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


def out_error(got_bf16: torch.Tensor, want_u16: np.ndarray):
    got = got_bf16.detach().float().cpu().numpy().astype(np.float64)
    want = oracle.bf16_to_f32(want_u16).astype(np.float64).reshape(got.shape)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300)
    rms = np.sqrt(np.mean(want ** 2))
    mx = np.abs(got - want).max() / max(rms, 1e-300)
    return rel, mx


def assert_out_close(got_bf16, want_u16, what=""):
    rel, mx = out_error(got_bf16, want_u16)
    assert rel <= REL_L2 and mx <= MAX_ABS_RMS, f"{what}: rel_l2={rel:.3e} max/rms={mx:.3e}"
    return rel, mx


def oracle_layer(cfg, inp, tokens=None, expert=None):
    """Oracle forward of the layer on the tokens listed (default all).  Tokens
    of an MoE layer are independent, so a subset is evaluated as its own batch."""
    x = inp["x"] if tokens is None else inp["x"][torch.as_tensor(tokens, device=inp["x"].device)]
    if expert is None:
        expert = lambda e: (u16(inp["w13"][e]), u16(inp["w2"][e]))
    return oracle.moe_layer(u16(x), u16(inp["w_router"]), inp["bias"].detach().cpu().numpy(),
                            expert, n_experts=cfg.n_experts, top_k=cfg.top_k,
                            n_shared=cfg.n_shared, precision=cfg.precision,
                            routed_scale=cfg.routed_scale)
