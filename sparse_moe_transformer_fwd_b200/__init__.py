"""B200 (sm_100a) forward pass of one DeepSeek-V3/R1 Mixture-of-Experts FFN
layer: sigmoid-affinity router with a routing-only bias and top-k, per-expert
permutation, blockwise e4m3 quantisation, grouped SwiGLU expert GEMMs on the
tcgen05 tensor cores, and a weighted combine with the always-on shared
expert.  The work happens in libmoe_fwd.so (include/moe_fwd.h); this package
is its binding.

    layer = MoELayer(w_router, bias, w13, w2, top_k=8, precision="fp8")
    out = layer(x)          # x: bf16 [T, d_model] on the GPU
"""
from __future__ import annotations

import torch

from ._native import (EXPORTS, MOE_BF16, MOE_FP8_BLOCK, MOE_FP8_UE8M0, MOE_LAYOUT_ROWMAJOR, MOE_LAYOUT_TILED,
                      MoeError, moe_pack_tiles, moe_forward_prenorm, MoeShape, alloc_workspace,
                      fp8_block_quant, lib, make_shape, moe_check_status, moe_combine,
                      moe_forward, moe_grouped_swiglu, moe_last_error, moe_last_launch_count,
                      moe_last_launch_names,
                      moe_permute, moe_route, moe_route_noalloc, moe_set_kernel_events,
                      moe_workspace_size, MOE_ROUTE_NOALLOC_MAX_SCORES, MoeDenseShape,
                      make_dense_shape, moe_dense_workspace_size, alloc_dense_workspace,
                      moe_dense_ffn, moe_dense_ffn_prenorm, moe_workspace_layout,
                      moe_quant_scatter, moe_ep_dispatch, moe_ep_workspace_size,
                      moe_ep_grouped_swiglu, MOE_EP_MAX_RANKS)

__all__ = [
    "MoELayer", "MoeError", "MoeShape", "make_shape", "alloc_workspace", "lib", "EXPORTS",
    "moe_workspace_size", "moe_route", "moe_permute", "fp8_block_quant", "moe_grouped_swiglu",
    "moe_combine", "moe_forward", "moe_check_status", "moe_last_error", "moe_last_launch_count",
    "quantize_weights", "MOE_BF16", "MOE_FP8_BLOCK", "MOE_FP8_UE8M0", "moe_set_kernel_events",
    "moe_route_noalloc", "MOE_ROUTE_NOALLOC_MAX_SCORES", "moe_pack_tiles", "pack_weights",
    "MOE_LAYOUT_ROWMAJOR", "MOE_LAYOUT_TILED", "moe_forward_prenorm", "moe_last_launch_names",
    "DenseFFN", "MoeDenseShape", "make_dense_shape", "moe_dense_workspace_size",
    "alloc_dense_workspace", "moe_dense_ffn", "moe_dense_ffn_prenorm", "moe_workspace_layout",
    "moe_quant_scatter", "moe_ep_dispatch", "moe_ep_workspace_size", "moe_ep_grouped_swiglu",
    "MOE_EP_MAX_RANKS",
]


def quantize_weights(w13: torch.Tensor, w2: torch.Tensor, stream=None, ue8m0: bool = False,
                     layout=MOE_LAYOUT_TILED):
    """128x128 e4m3 block quantisation of the stacked expert weights (done
    once, ahead of the forward passes), codes in `layout` (tiled by default,
    or row-major); ue8m0: power-of-two scales.  Returns (w13q, w13s, w2q, w2s)."""
    S, n13, d = w13.shape
    _, d2, de = w2.shape
    w13q = torch.empty(S, n13, d, dtype=torch.uint8, device=w13.device)
    w13s = torch.empty(S, n13 // 128, d // 128, dtype=torch.float32, device=w13.device)
    w2q = torch.empty(S, d2, de, dtype=torch.uint8, device=w2.device)
    w2s = torch.empty(S, d2 // 128, de // 128, dtype=torch.float32, device=w2.device)
    fp8_block_quant(w13, 128, w13q, w13s, layout=layout, stream=stream, ue8m0=ue8m0)
    fp8_block_quant(w2, 128, w2q, w2s, layout=layout, stream=stream, ue8m0=ue8m0)
    return w13q, w13s, w2q, w2s


def pack_weights(w13: torch.Tensor, w2: torch.Tensor, stream=None):
    """bf16 expert weights repacked into the tiled layout the GEMMs read."""
    a, b = torch.empty_like(w13), torch.empty_like(w2)
    moe_pack_tiles(w13.contiguous(), a, stream=stream)
    moe_pack_tiles(w2.contiguous(), b, stream=stream)
    return a, b


class MoELayer:
    """One MoE FFN layer with resident weights.

    w_router bf16 [E, d]; bias fp32 [E]; w13 bf16 [E + n_shared, 2*d_expert, d]
    (gate rows then up rows); w2 bf16 [E + n_shared, d, d_expert]; the shared
    expert, if any, is the last slot.  precision "fp8" (fp32 block scales) or
    "fp8_ue8m0" (power-of-two block scales) quantises the expert weights once
    at construction (the bf16 copies are then not needed); "bf16" repacks
    them.  weight_layout "tiled" (default: 128 x 128-byte tiles, one
    contiguous 16 KB read per TMA box) or "rowmajor" (the weights as given,
    e4m3 codes row-major)."""

    def __init__(self, w_router, bias, w13, w2, *, top_k: int, n_shared: int = 1,
                 routed_scale: float = 1.0, precision: str = "fp8", keep_bf16: bool = False,
                 weight_layout: str = "tiled"):
        lib()  # fail loudly now if the CUDA library is missing
        self.E, self.d = w_router.shape
        self.de = w2.shape[2]
        self.top_k, self.n_shared, self.routed_scale = top_k, n_shared, routed_scale
        self.precision = precision
        if weight_layout not in ("tiled", "rowmajor"):
            raise ValueError(weight_layout)
        self.weight_layout = weight_layout
        lay = MOE_LAYOUT_TILED if weight_layout == "tiled" else MOE_LAYOUT_ROWMAJOR
        self.w_router, self.bias = w_router.contiguous(), bias.contiguous()
        if precision in ("fp8", "fp8_ue8m0"):
            self.w13, self.w13s, self.w2, self.w2s = quantize_weights(
                w13.contiguous(), w2.contiguous(), ue8m0=precision == "fp8_ue8m0", layout=lay)
            self.w13_bf16 = w13 if keep_bf16 else None
            self.w2_bf16 = w2 if keep_bf16 else None
        elif precision == "bf16":
            self.w13, self.w2 = pack_weights(w13, w2) if lay == MOE_LAYOUT_TILED else \
                (w13.contiguous(), w2.contiguous())
            self.w13s = self.w2s = None
        else:
            raise ValueError(precision)
        self._ws = {}

    def shape(self, T: int) -> MoeShape:
        return make_shape(T, self.d, self.E, self.top_k, self.de, self.n_shared,
                          self.routed_scale, self.precision, self.weight_layout)

    def workspace(self, T: int) -> torch.Tensor:
        ws = self._ws.get(T)
        if ws is None:
            ws = alloc_workspace(self.shape(T), self.w13.device)
            self._ws[T] = ws
        return ws

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None,
                 topk_idx_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if out is None:
            out = torch.empty(T, self.d, dtype=torch.bfloat16, device=x.device)
        moe_forward(self.shape(T), x, self.w_router, self.bias, self.w13, self.w13s, self.w2,
                    self.w2s, out, self.workspace(T), topk_idx_out=topk_idx_out, stream=stream)
        return out

    def forward_prenorm(self, h: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
                        out: torch.Tensor | None = None,
                        topk_idx_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """The FFN block: out = h + MoE(RMSNorm(h) * gamma) (pre-norm fused)."""
        T = h.shape[0]
        if out is None:
            out = torch.empty(T, self.d, dtype=torch.bfloat16, device=h.device)
        moe_forward_prenorm(self.shape(T), h, gamma, eps, self.w_router, self.bias, self.w13,
                            self.w13s, self.w2, self.w2s, out, self.workspace(T),
                            topk_idx_out=topk_idx_out, stream=stream)
        return out

    def check_status(self, T: int) -> int:
        return moe_check_status(self.workspace(T))


class DenseFFN:
    """One dense gated FFN layer (the model's first layers) with resident
    weights, on the expert GEMM kernels.

    w13 bf16 [2*d_ff, d] (gate rows then up rows); w2 bf16 [d, d_ff].
    precision and weight_layout as for MoELayer."""

    def __init__(self, w13, w2, *, precision: str = "fp8", weight_layout: str = "tiled"):
        lib()
        self.d, self.d_ff = w2.shape
        self.precision = precision
        if weight_layout not in ("tiled", "rowmajor"):
            raise ValueError(weight_layout)
        self.weight_layout = weight_layout
        lay = MOE_LAYOUT_TILED if weight_layout == "tiled" else MOE_LAYOUT_ROWMAJOR
        w13, w2 = w13.contiguous().unsqueeze(0), w2.contiguous().unsqueeze(0)
        if precision in ("fp8", "fp8_ue8m0"):
            self.w13, self.w13s, self.w2, self.w2s = quantize_weights(
                w13, w2, ue8m0=precision == "fp8_ue8m0", layout=lay)
        elif precision == "bf16":
            self.w13, self.w2 = pack_weights(w13, w2) if lay == MOE_LAYOUT_TILED else (w13, w2)
            self.w13s = self.w2s = None
        else:
            raise ValueError(precision)
        self._ws = {}

    def shape(self, T: int) -> MoeDenseShape:
        return make_dense_shape(T, self.d, self.d_ff, self.precision, self.weight_layout)

    def workspace(self, T: int) -> torch.Tensor:
        ws = self._ws.get(T)
        if ws is None:
            ws = alloc_dense_workspace(self.shape(T), self.w13.device)
            self._ws[T] = ws
        return ws

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        T = x.shape[0]
        if out is None:
            out = torch.empty(T, self.d, dtype=torch.bfloat16, device=x.device)
        moe_dense_ffn(self.shape(T), x, self.w13, self.w13s, self.w2, self.w2s, out,
                      self.workspace(T), stream=stream)
        return out

    def forward_prenorm(self, h: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
                        out: torch.Tensor | None = None, stream=None):
        """The FFN block: out = h + FFN(RMSNorm(h) * gamma)."""
        T = h.shape[0]
        if out is None:
            out = torch.empty(T, self.d, dtype=torch.bfloat16, device=h.device)
        moe_dense_ffn_prenorm(self.shape(T), h, gamma, eps, self.w13, self.w13s, self.w2,
                              self.w2s, out, self.workspace(T), stream=stream)
        return out

    def check_status(self, T: int) -> int:
        return moe_check_status(self.workspace(T))
