"""The expert-parallel layer on one GPU: G = 2 and 4 ranks whose buffers all
live on this device, run stream-ordered (moe_route, moe_permute,
moe_quant_scatter per rank; moe_ep_dispatch into the owners' receive
buffers; moe_ep_grouped_swiglu over (source, expert) segments with Y stored
back into the sources' buffers by the down GEMM; the shared expert; the
combine).  Checked against:
  - the oracle's data-parallel layer on each rank's tokens (output
    tolerance, routing bit-exact);
  - the receive buffers: every source's rows and scales, bit for bit, where
    the exchange plan puts them;
  - the library's data-parallel forward on the same tokens, bit for bit
    where both run 128-row tiles (the rows of a segment meet the same
    arithmetic whichever rank computes them).
"Local Balanced Routing to Experts" ("DeepSeek v3 and R1 Model
Architecture"): experts spread over devices, tokens sent to them."""
import numpy as np
import pytest
import torch

import sparse_moe_transformer_fwd_b200 as moe
from moe_inputs import CONFIGS, make_inputs
from sparse_moe_transformer_fwd_b200.ep import EPShard, ep_forward_emulated
from sparse_moe_transformer_fwd_b200.ep_plan import dispatch_blocks

from _gpu_util import assert_out_close, oracle_layer

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None

CASES = {
    # name: (base config, world, tokens per rank)
    "tiny_G2": ("tiny", 2, [100, 37]),
    "tiny_G4": ("tiny", 4, [130, 64, 5, 77]),
    "tiny_G4_empty_rank": ("tiny", 4, [90, 0, 33, 129]),
    "ds_G4": ("decode", 4, [96, 64, 130, 80]),
}


def _shards(cfg, inp, G):
    P = cfg.n_experts // G
    return [EPShard(inp["w_router"], inp["bias"], inp["w13"][r * P:(r + 1) * P],
                    inp["w2"][r * P:(r + 1) * P], inp["w13"][cfg.n_experts],
                    inp["w2"][cfg.n_experts], n_experts=cfg.n_experts, top_k=cfg.top_k, rank=r,
                    world=G, precision=cfg.precision) for r in range(G)]


@pytest.mark.parametrize("precision", ["fp8", "bf16", "fp8_ue8m0"])
@pytest.mark.parametrize("name", list(CASES))
def test_ep_forward_matches_data_parallel(name, precision):
    base, G, Ts = CASES[name]
    if base == "decode" and precision != "fp8":
        pytest.skip("DeepSeek dims: the fp32-scale workload only")
    cfg = CONFIGS[base].with_(precision=precision, T=sum(Ts))
    inp = make_inputs(cfg, seed=21, device=DEV)
    xs = list(torch.split(inp["x"], Ts))
    shards = _shards(cfg, inp, G)
    outs, states, recv_a, recv_s, plans = ep_forward_emulated(shards, xs, keep=True)
    for st in states:
        assert moe.moe_check_status(st["ws"]) == 0, moe.moe_last_error()
        if "shared_ws" in st:
            assert moe.moe_check_status(st["shared_ws"]) == 0, moe.moe_last_error()
    for sh in shards:
        if hasattr(sh, "_last_ws"):
            assert moe.moe_check_status(sh._last_ws) == 0, moe.moe_last_error()
    # receive buffers: each source's block where the plan puts it
    counts_all = np.stack([st["counts"].cpu().numpy() for st in states])
    for s in range(G):
        for src_row, rows, o, dst_row in dispatch_blocks(counts_all, s):
            a = states[s]["a"][src_row:src_row + rows]
            assert torch.equal(recv_a[o][dst_row:dst_row + rows].view(torch.uint8),
                               a.view(torch.uint8))
            if recv_s is not None:
                assert torch.equal(recv_s[o][dst_row:dst_row + rows].view(torch.int32),
                                   states[s]["a_scales"][src_row:src_row + rows].view(torch.int32))
    # the library's data-parallel forward on each rank's tokens
    dp = moe.MoELayer(inp["w_router"], inp["bias"], inp["w13"], inp["w2"], top_k=cfg.top_k,
                      n_shared=1, precision=precision)
    for r, (x, out) in enumerate(zip(xs, outs)):
        T = x.shape[0]
        if T == 0:
            assert out.shape == (0, cfg.d_model)
            continue
        idx = torch.empty(T, cfg.top_k, dtype=torch.int32, device=DEV)
        ref_out = dp(x, topk_idx_out=idx)
        assert torch.equal(states[r]["idx"], idx)
        # 64-row tiles (fp32 scales, at most 64 tokens) sum K in another order
        if not (precision == "fp8" and T <= 64):
            assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), f"rank {r}"
        ref = oracle_layer(cfg.with_(T=T), {**inp, "x": x})
        assert np.array_equal(states[r]["idx"].cpu().numpy(), ref["idx"])
        assert_out_close(out, ref["out"], f"EP {name} {precision} rank {r}", ref["out_allow"])


def test_ep_bad_segment_reports_status():
    """A segment that would return rows past its source's buffer is recorded
    in the workspace status word and skipped; the context stays usable."""
    cfg = CONFIGS["tiny"].with_(precision="fp8")
    inp = make_inputs(cfg, seed=22, device=DEV)
    shard = _shards(cfg, inp, 1)[0]
    T = 40
    st = shard.prepare(inp["x"][:T])
    i32 = lambda v: torch.tensor(v, dtype=torch.int32, device=DEV)
    ws = torch.zeros(moe.moe_ep_workspace_size(st["shape"], st["a"].shape[0], 2),
                     dtype=torch.uint8, device=DEV)
    small_y = torch.empty(8, cfg.d_model, dtype=torch.bfloat16, device=DEV)
    moe.moe_ep_grouped_swiglu(st["shape"], st["a"], st["a_scales"], i32([0, 10]), i32([10, 20]),
                              i32([0, 1]), i32([0, 0]), i32([0, 0]), cfg.n_experts, shard.w13,
                              shard.w13s, shard.w2, shard.w2s, [small_y], ws)
    assert moe.moe_check_status(ws) == moe._native.MOE_ERR_DEVICE_INDEX
    assert moe.moe_check_status(ws) == 0
    torch.cuda.synchronize()
