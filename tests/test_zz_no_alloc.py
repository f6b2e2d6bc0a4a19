"""moe_route_noalloc: the router for callers that may not allocate device
memory (no cudaMalloc, no workspace; e.g. code inside a framework plugin that
owns all device memory, or a serving loop that forbids allocation after
start-up).  Its score scratch is a fixed array inside the library.  Checked
through the C ABI against moe_route on the same inputs, bit for bit (routing
is compared exactly everywhere in this suite), on two calls in a row; and the
size limit is enforced before anything is enqueued.

Kept in a file that sorts last so that a run stopping at its first failure
has already run every other test."""
import numpy as np
import pytest
import torch

import sparse_moe_transformer_fwd_b200 as moe
from moe_inputs import CONFIGS, make_x, make_router

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def _route_both(cfg, seed):
    x = make_x(cfg, seed, "cpu").to(DEV)
    w, b = make_router(cfg, seed, "cpu")
    w, b = w.to(DEV), b.to(DEV)
    shape = moe.make_shape(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_expert,
                           cfg.n_shared, cfg.routed_scale, cfg.precision)
    ws = moe.alloc_workspace(shape, DEV)
    idx_ref = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=DEV)
    g_ref = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=DEV)
    moe.moe_route(shape, x, w, b, idx_ref, g_ref, ws)
    assert moe.moe_check_status(ws) == 0
    outs = []
    for _ in range(2):  # two calls in a row share the fixed scratch
        idx = torch.full((cfg.T, cfg.top_k), -1, dtype=torch.int32, device=DEV)
        g = torch.full((cfg.T, cfg.top_k), -1.0, dtype=torch.float32, device=DEV)
        moe.moe_route_noalloc(shape, x, w, b, idx, g)
        torch.cuda.synchronize()
        outs.append((idx.cpu(), g.cpu()))
    return (idx_ref.cpu(), g_ref.cpu()), outs


@pytest.mark.parametrize("name,T", [("decode", 64), ("tiny", 128), ("decode", 4096)])
def test_noalloc_route_matches_moe_route(name, T):
    cfg = CONFIGS[name].with_(T=T)
    (idx_ref, g_ref), outs = _route_both(cfg, seed=5)
    for idx, g in outs:
        assert torch.equal(idx, idx_ref)
        assert np.array_equal(g.numpy().view(np.uint32), g_ref.numpy().view(np.uint32))


def test_noalloc_route_rejects_oversize():
    cfg = CONFIGS["decode"].with_(T=moe.MOE_ROUTE_NOALLOC_MAX_SCORES // 256 + 1)
    shape = moe.make_shape(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_expert)
    t = torch.empty(16, dtype=torch.int32, device=DEV)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_route_noalloc(shape, t.view(torch.bfloat16), t.view(torch.bfloat16),
                              t.float(), t, t.float())
    assert ei.value.code == moe._native.MOE_ERR_INVALID_ARG
    assert "exceeds" in moe.moe_last_error()
