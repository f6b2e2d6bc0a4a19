"""The forward passes can be captured in a CUDA graph: every call only
enqueues kernels (no synchronisation, no allocation, programmatic-dependent
launches between them), so a graph of the MoE layer or of the dense layer
replays the same launches.  Replays with new inputs copied into the captured
input buffer give the eager results bit for bit, and the status word stays
clean."""
import pytest
import torch

import sparse_moe_transformer_fwd_b200 as moe
from moe_inputs import CONFIGS, DENSE_CONFIGS, make_dense_inputs, make_inputs, make_residual
from moe_inputs import make_x

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def _replays_match(call, x_static, out_static, cfg, T):
    call(x_static, out_static)  # warm-up: workspace allocated, attributes set
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(x_static, out_static)
    for seed in (5, 6, 7):
        x_new = make_x(cfg, seed=seed, T=T).to(DEV)
        want = torch.empty_like(out_static)
        call(x_new, want)
        x_static.copy_(x_new)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_static.view(torch.int16), want.view(torch.int16)), seed
    del g


@pytest.mark.parametrize("name,precision,T", [("tiny", "bf16", 100), ("tiny", "fp8", 64),
                                              ("tiny", "fp8", 300), ("tiny", "fp8_ue8m0", 64),
                                              ("decode_small", "fp8", 64)])
def test_moe_forward_graph_replay(name, precision, T):
    cfg = CONFIGS[name].with_(precision=precision, T=T)
    inp = {k: v.to(DEV) for k, v in make_inputs(cfg, seed=4).items()}
    layer = moe.MoELayer(inp["w_router"], inp["bias"], inp["w13"], inp["w2"], top_k=cfg.top_k,
                         precision=precision)
    x_static = inp["x"].clone()
    out_static = torch.empty(T, cfg.d_model, dtype=torch.bfloat16, device=DEV)
    _replays_match(lambda x, o: layer(x, out=o), x_static, out_static, cfg, T)
    assert layer.check_status(T) == 0


def test_moe_prenorm_graph_replay():
    cfg = CONFIGS["tiny"].with_(precision="fp8", T=48)
    inp = {k: v.to(DEV) for k, v in make_inputs(cfg, seed=4).items()}
    layer = moe.MoELayer(inp["w_router"], inp["bias"], inp["w13"], inp["w2"], top_k=cfg.top_k,
                         precision="fp8")
    h, gamma = make_residual(cfg, seed=4, device=DEV)
    out_static = torch.empty_like(h)
    _replays_match(lambda x, o: layer.forward_prenorm(x, gamma, out=o), h.clone(), out_static,
                   cfg, cfg.T)
    assert layer.check_status(cfg.T) == 0


@pytest.mark.parametrize("precision,T", [("fp8", 48), ("fp8", 300), ("bf16", 100)])
def test_dense_graph_replay(precision, T):
    cfg = DENSE_CONFIGS["dense_tiny"].with_(precision=precision, T=T)
    inp = {k: v.to(DEV) for k, v in make_dense_inputs(cfg, seed=4).items()}
    layer = moe.DenseFFN(inp["w13"], inp["w2"], precision=precision)
    out_static = torch.empty(T, cfg.d_model, dtype=torch.bfloat16, device=DEV)
    _replays_match(lambda x, o: layer(x, out=o), inp["x"].clone(), out_static, cfg, T)
    assert layer.check_status(T) == 0
