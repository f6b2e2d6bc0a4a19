"""Expert-parallel MoE layer ("DeepSeek v3 and R1 Model Architecture", "Local
Balanced Routing to Experts": routed experts spread over devices, tokens
sent to the devices that hold their experts).

G ranks; rank r owns routed experts r*P .. r*P + P - 1 (P = E / G) and every
rank holds the router and the shared expert.  EPShard is one rank's part;
ep_forward_emulated runs the layer for G ranks whose buffers all live on the
current GPU (every step stream-ordered on one stream; no flags between
kernels), the form a single GPU can execute and test.  On several GPUs the
same library calls run one rank per process, with the receive and Y buffers
of the other ranks given as peer-mapped pointers and the counts exchanged by
ep_plan.exchange_counts.

The steps of one call (include/moe_fwd.h, "Expert parallelism"):
  every rank: moe_route, moe_permute, moe_quant_scatter on its own tokens;
  counts of all ranks -> exchange plan (ep_plan);
  every source: moe_ep_dispatch of its block for each owner;
  every owner: moe_ep_grouped_swiglu over (source, local expert) segments,
      the down GEMM storing each Y row into its source's Y buffer;
  every rank: moe_ep_grouped_swiglu over its shared rows, moe_combine.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _native as N
from .ep_plan import dispatch_blocks, ep_plan, gemm_segments

__all__ = ["EPShard", "ep_forward_emulated"]


class EPShard:
    """One rank's part of an expert-parallel MoE layer.

    w_router bf16 [E, d], bias fp32 [E] (replicated); w13_local bf16
    [P, 2*d_expert, d] and w2_local bf16 [P, d, d_expert] (this rank's routed
    experts, global index rank*P + i in slot i); w13_shared / w2_shared the
    shared expert ([2*d_expert, d], [d, d_expert]).  Weights are quantised
    (fp8 precisions) or repacked (bf16) once, as in MoELayer."""

    def __init__(self, w_router, bias, w13_local, w2_local, w13_shared, w2_shared, *,
                 n_experts: int, top_k: int, rank: int, world: int, precision: str = "fp8",
                 routed_scale: float = 1.0, weight_layout: str = "tiled"):
        from . import pack_weights, quantize_weights
        N.lib()
        if n_experts % world or w13_local.shape[0] != n_experts // world:
            raise ValueError("each rank holds n_experts / world routed experts")
        self.E, self.d = w_router.shape
        self.de = w2_local.shape[2]
        self.k, self.rank, self.world = top_k, rank, world
        self.precision, self.routed_scale, self.weight_layout = precision, routed_scale, weight_layout
        self.w_router, self.bias = w_router.contiguous(), bias.contiguous()
        lay = N.MOE_LAYOUT_TILED if weight_layout == "tiled" else N.MOE_LAYOUT_ROWMAJOR
        sh13, sh2 = w13_shared.contiguous().unsqueeze(0), w2_shared.contiguous().unsqueeze(0)
        if precision in ("fp8", "fp8_ue8m0"):
            ue = precision == "fp8_ue8m0"
            self.w13, self.w13s, self.w2, self.w2s = quantize_weights(
                w13_local.contiguous(), w2_local.contiguous(), ue8m0=ue, layout=lay)
            self.sw13, self.sw13s, self.sw2, self.sw2s = quantize_weights(sh13, sh2, ue8m0=ue,
                                                                          layout=lay)
        elif precision == "bf16":
            if lay == N.MOE_LAYOUT_TILED:
                self.w13, self.w2 = pack_weights(w13_local, w2_local)
                self.sw13, self.sw2 = pack_weights(sh13, sh2)
            else:
                self.w13, self.w2 = w13_local.contiguous(), w2_local.contiguous()
                self.sw13, self.sw2 = sh13, sh2
            self.w13s = self.w2s = self.sw13s = self.sw2s = None
        else:
            raise ValueError(precision)

    @property
    def fp8(self) -> bool:
        return self.precision != "bf16"

    def shape(self, T: int):
        return N.make_shape(T, self.d, self.E, self.k, self.de, 1, self.routed_scale,
                            self.precision, self.weight_layout)

    def prepare(self, x: torch.Tensor, stream=None) -> dict:
        """Steps on the rank's own tokens: routing, permutation and the
        permuted (quantised) rows, in buffers of this rank."""
        T, dev = x.shape[0], x.device
        shape = self.shape(T)
        ws = N.alloc_workspace(shape, dev)
        st = {"T": T, "shape": shape, "ws": ws, "x": x}
        st["idx"] = torch.empty(T, self.k, dtype=torch.int32, device=dev)
        st["gates"] = torch.empty(T, self.k, dtype=torch.float32, device=dev)
        st["counts"] = torch.empty(self.E, dtype=torch.int32, device=dev)
        st["offsets"] = torch.empty(self.E + 1, dtype=torch.int32, device=dev)
        st["row_token"] = torch.empty(T * self.k, dtype=torch.int32, device=dev)
        st["row_of"] = torch.empty(T, self.k, dtype=torch.int32, device=dev)
        R_s = T * (self.k + 1)
        st["a"] = torch.empty(R_s, self.d, dtype=torch.uint8 if self.fp8 else torch.bfloat16,
                              device=dev)
        st["a_scales"] = (torch.empty(R_s, self.d // 128, dtype=torch.float32, device=dev)
                          if self.fp8 else None)
        st["y"] = torch.empty(R_s, self.d, dtype=torch.bfloat16, device=dev)
        if T == 0:
            st["counts"].zero_()
            return st
        N.moe_route(shape, x, self.w_router, self.bias, st["idx"], st["gates"], ws, stream)
        N.moe_permute(shape, st["idx"], st["counts"], st["offsets"], st["row_token"], st["row_of"],
                      ws, stream)
        N.moe_quant_scatter(shape, x, st["row_of"], st["a"], st["a_scales"], stream)
        return st


def ep_forward_emulated(shards, xs, stream=None, keep=False):
    """Expert-parallel forward of len(shards) ranks whose buffers all live on
    this GPU.  xs[r]: rank r's tokens, bf16 [T_r, d].  Returns each rank's
    output (bf16 [T_r, d]); keep=True also returns the per-rank state and the
    receive buffers.  The one host synchronisation is the count exchange,
    which sizes the receive buffers."""
    G = len(shards)
    dev = xs[0].device
    states = [sh.prepare(x, stream) for sh, x in zip(shards, xs)]
    counts_all = torch.stack([s["counts"] for s in states]).cpu().numpy()
    plans = [ep_plan(counts_all, o) for o in range(G)]
    sh0 = shards[0]
    recv_a = [torch.empty(max(p.total_recv, 1), sh0.d,
                          dtype=torch.uint8 if sh0.fp8 else torch.bfloat16, device=dev)
              for p in plans]
    recv_s = ([torch.empty(max(p.total_recv, 1), sh0.d // 128, dtype=torch.float32, device=dev)
               for p in plans] if sh0.fp8 else None)
    for s in range(G):
        blocks = dispatch_blocks(counts_all, s)
        if blocks:
            N.moe_ep_dispatch(states[s]["shape"], states[s]["a"], states[s]["a_scales"], blocks,
                              recv_a, recv_s, stream)
    ret_y = [st["y"] for st in states]
    for o in range(G):
        if plans[o].total_recv == 0:
            continue
        sg = {k: torch.from_numpy(v).to(dev) for k, v in gemm_segments(plans[o]).items()}
        sh = shards[o]
        shape = sh.shape(states[o]["T"])
        rows = plans[o].total_recv
        ws = torch.zeros(N.moe_ep_workspace_size(shape, rows, sg["seg_start"].numel()),
                         dtype=torch.uint8, device=dev)
        N.moe_ep_grouped_swiglu(shape, recv_a[o][:rows], recv_s[o][:rows] if recv_s else None,
                                sg["seg_start"], sg["seg_rows"], sg["seg_slot"], sg["seg_src"],
                                sg["seg_ret"], sh.E // sh.world, sh.w13, sh.w13s, sh.w2, sh.w2s,
                                ret_y, ws, stream)
        sh._last_ws = ws
    outs = []
    for r, (sh, st) in enumerate(zip(shards, states)):
        T = st["T"]
        out = torch.empty(T, sh.d, dtype=torch.bfloat16, device=dev)
        if T == 0:
            outs.append(out)
            continue
        # the shared expert on the rank's own shared rows (T*k .. T*k+T-1)
        one = lambda v: torch.tensor([v], dtype=torch.int32, device=dev)
        ws = torch.zeros(N.moe_ep_workspace_size(st["shape"], st["a"].shape[0], 1),
                         dtype=torch.uint8, device=dev)
        N.moe_ep_grouped_swiglu(st["shape"], st["a"], st["a_scales"], one(T * sh.k), one(T), one(0),
                                one(0), one(T * sh.k), 1, sh.sw13, sh.sw13s, sh.sw2, sh.sw2s,
                                [st["y"]], ws, stream)
        st["shared_ws"] = ws
        N.moe_combine(st["shape"], st["y"], st["row_of"], st["gates"], out, stream)
        outs.append(out)
    if keep:
        return outs, states, recv_a, recv_s, plans
    return outs
