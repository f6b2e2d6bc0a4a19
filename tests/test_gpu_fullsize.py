"""GPU parity at the full DeepSeek-V3 layer sizes (d_model 7168, 256 experts
top-8 + 1 shared, d_expert 2048) for the decode (T=64), prefill (T=4096),
skewed-routing (T=16384) and bf16 (T=8192) workloads and the UE8M0 variants,
in the launch configuration the benchmark times (one moe_forward call).

What is compared, per workload:
  - routing of EVERY token: the affinities s [T, E], the expert indices and
    the gates bit for bit against the oracle's router run on all T tokens
    ("DeepSeek v3 and R1 Model Architecture", "Local Balanced Routing to
    Experts": selection by affinity plus a routing-only bias);
  - the permutation the forward itself built (counts, offsets, row_token,
    row_of, read from its workspace) bit for bit against the oracle's
    permutation of the oracle's indices;
  - the permuted activations the grouped GEMM read: e4m3 codes and fp32
    scales (bf16 rows in the bf16 workload) bit for bit against the
    oracle's 1x128 quantisation of x gathered by the oracle's row_token
    ("DeepSeek-R1", "Quantization": blockwise FP8);
  - the 128x128 weight codes and scales of three experts bit for bit;
  - the output rows of a 512-token sample (all tokens when T <= 512) that
    covers every expert some token chose: each expert's last token (a row of
    its last, ragged tile), the hottest expert's last 16 and first 4 tokens,
    tokens 0 and T-1 (the shared segment's ends), then seeded draws; within
    the output tolerance against the oracle's expert math on those tokens.
Inputs are generated on the GPU by the seeded generators; the oracle gets
host copies.  The oracle's router and experts run on several host threads
(each step single-threaded, results independent of the split)."""
import os

import numpy as np
import pytest
import torch

import oracle
import sparse_moe_transformer_fwd_b200 as moe
from moe_inputs import CONFIGS, make_inputs

from _gpu_util import assert_out_close, u16, untile

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None
WORKERS = max(1, min(len(os.sched_getaffinity(0)), 32))
N_SAMPLE = 512


def coverage_sample(idx: np.ndarray, n_experts: int, n: int = N_SAMPLE, seed: int = 0):
    """Tokens whose output rows are compared (sorted): every token when
    T <= n; else the last token of every expert with tokens (segments hold
    their tokens in ascending order, so that row is in the expert's last
    tile), the hottest expert's last 16 and first 4 tokens, tokens 0 and
    T-1, and seeded uniform draws up to n."""
    T = idx.shape[0]
    if T <= n:
        return np.arange(T)
    sel = {0, T - 1}
    counts = np.bincount(idx.reshape(-1), minlength=n_experts)
    for e in np.nonzero(counts)[0]:
        sel.add(int(np.nonzero((idx == e).any(1))[0][-1]))
    hot = int(np.argmax(counts))
    toks = np.nonzero((idx == hot).any(1))[0]
    sel.update(int(t) for t in toks[-16:])
    sel.update(int(t) for t in toks[:4])
    rng = np.random.default_rng(seed)
    while len(sel) < n:
        sel.add(int(rng.integers(T)))
    return np.array(sorted(sel))


def _ws_region(ws, off, name, count, dtype):
    item = torch.tensor([], dtype=dtype).element_size()
    return ws[off[name]:off[name] + count * item].view(dtype).cpu().numpy()


@pytest.fixture(scope="module", params=["decode", "prefill", "skew", "bf16", "decode_ue8m0",
                                        "prefill_ue8m0"])
def run(request):
    cfg = CONFIGS[request.param]
    T, E, k, d = cfg.T, cfg.n_experts, cfg.top_k, cfg.d_model
    inp = make_inputs(cfg, seed=0, device=DEV)
    layer = moe.MoELayer(inp["w_router"], inp["bias"], inp["w13"], inp["w2"], top_k=k,
                         n_shared=cfg.n_shared, precision=cfg.precision)
    out = layer(inp["x"])          # indices stay in the workspace (topk_idx_out NULL)
    status = layer.check_status(T)
    # the forward's own intermediate results, copied out of its workspace
    shape = layer.shape(T)
    off = moe.moe_workspace_layout(shape)
    ws = layer.workspace(T)
    Rs = cfg.R_s
    fp8 = cfg.precision != "bf16"
    gpu = {
        "scores": _ws_region(ws, off, "scores", T * E, torch.float32).reshape(T, E),
        "idx": _ws_region(ws, off, "topk_idx", T * k, torch.int32).reshape(T, k),
        "gates": _ws_region(ws, off, "topk_w", T * k, torch.float32).reshape(T, k),
        "counts": _ws_region(ws, off, "counts", E, torch.int32),
        "offsets": _ws_region(ws, off, "offsets", E + 1, torch.int32),
        "row_token": _ws_region(ws, off, "row_token", T * k, torch.int32),
        "row_of": _ws_region(ws, off, "row_of", T * k, torch.int32).reshape(T, k),
    }
    if fp8:
        gpu["a"] = _ws_region(ws, off, "a", Rs * d, torch.uint8).reshape(Rs, d)
        gpu["a_scales"] = _ws_region(ws, off, "a_scales", Rs * (d // 128),
                                     torch.float32).reshape(Rs, d // 128)
    else:
        gpu["a"] = _ws_region(ws, off, "a", Rs * d, torch.int16).view(np.uint16).reshape(Rs, d)
    # the oracle's router on every token
    x_h = u16(inp["x"])
    logits = oracle.router_logits(x_h, u16(inp["w_router"]), workers=WORKERS)
    ref = dict(zip(("idx", "gates", "scores"),
                   oracle.route(logits, inp["bias"].cpu().numpy(), k, cfg.routed_scale)))
    yield cfg, inp, layer, out, status, gpu, ref, x_h
    del layer, inp, out, gpu
    torch.cuda.empty_cache()


def test_status_ok(run):
    assert run[4] == 0, moe.moe_last_error()


def test_routing_every_token_bitexact(run):
    """Affinities, indices and gates of all T tokens, bit for bit."""
    cfg, gpu, ref = run[0], run[5], run[6]
    assert np.array_equal(gpu["scores"].view(np.uint32), ref["scores"].view(np.uint32))
    assert np.array_equal(gpu["idx"], ref["idx"])
    assert np.array_equal(gpu["gates"].view(np.uint32), ref["gates"].view(np.uint32))
    if cfg.name == "skew":   # the hottest expert carries about 10x the mean load
        counts = np.bincount(ref["idx"].reshape(-1), minlength=cfg.n_experts)
        ratio = counts.max() / (cfg.T * cfg.top_k / cfg.n_experts)
        assert 8.0 <= ratio <= 12.0, ratio


def test_permutation_bitexact(run):
    """The forward's permutation against the oracle's, on the oracle's indices."""
    cfg, gpu, ref = run[0], run[5], run[6]
    rc, ro, rt, rr = oracle.permute(ref["idx"], cfg.n_experts)
    assert np.array_equal(gpu["counts"], rc)
    assert np.array_equal(gpu["offsets"], ro)
    assert np.array_equal(gpu["row_token"], rt)
    assert np.array_equal(gpu["row_of"], rr)


def test_permuted_activations_bitexact(run):
    """Rows the grouped GEMM read: routed rows are x[row_token] quantised
    1x128 (codes and scales), then the shared segment, x in token order."""
    cfg, gpu, ref, x_h = run[0], run[5], run[6], run[7]
    _, _, rt, _ = oracle.permute(ref["idx"], cfg.n_experts)
    order = np.concatenate([rt, np.arange(cfg.T, dtype=rt.dtype)])
    if cfg.precision == "bf16":
        assert np.array_equal(gpu["a"], x_h[order])
        return
    q, sc = oracle.block_quant(x_h, 1, ue8m0=cfg.precision == "fp8_ue8m0")
    assert np.array_equal(gpu["a"], q[order])
    assert np.array_equal(gpu["a_scales"].view(np.uint32), sc[order].view(np.uint32))


def test_weight_quant_bitexact(run):
    cfg, inp, layer = run[:3]
    if cfg.precision == "bf16":
        pytest.skip("bf16 workload: the weights are not quantised")
    ue = cfg.precision == "fp8_ue8m0"
    for e in (0, 137 % cfg.n_experts, cfg.n_experts):
        q13, s13 = oracle.block_quant(u16(inp["w13"][e]), 128, ue8m0=ue)
        assert np.array_equal(layer.w13s[e].cpu().numpy().view(np.uint32), s13.view(np.uint32))
        assert np.array_equal(untile(layer.w13[e].cpu().numpy(), *q13.shape), q13)
        q2, s2 = oracle.block_quant(u16(inp["w2"][e]), 128, ue8m0=ue)
        assert np.array_equal(layer.w2s[e].cpu().numpy().view(np.uint32), s2.view(np.uint32))
        assert np.array_equal(untile(layer.w2[e].cpu().numpy(), *q2.shape), q2)


def test_sampled_outputs_vs_oracle(run):
    """Output rows of the coverage sample within tolerance; the sample covers
    every expert that some token chose."""
    cfg, inp, layer, out, _, gpu, ref, x_h = run
    tokens = coverage_sample(ref["idx"], cfg.n_experts)
    chosen = set(np.unique(ref["idx"]).tolist())
    assert chosen <= set(np.unique(ref["idx"][tokens]).tolist())

    def expert(e):
        # host copies on demand (the oracle quantises them itself)
        return u16(inp["w13"][e]), u16(inp["w2"][e])

    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        res = oracle.moe_layer(x_h[tokens], u16(inp["w_router"]), inp["bias"].cpu().numpy(),
                               expert, n_experts=cfg.n_experts, top_k=cfg.top_k,
                               n_shared=cfg.n_shared, precision=cfg.precision,
                               routed_scale=cfg.routed_scale, workers=min(WORKERS, 16))
    assert np.array_equal(res["idx"], ref["idx"][tokens])
    assert_out_close(out[torch.as_tensor(tokens, device=DEV)], res["out"],
                     f"{cfg.name} sample of {len(tokens)} tokens", res["out_allow"])


def test_prenorm_decode_fullsize():
    """The pre-norm block at the decode batch and DeepSeek dims, as the
    benchmark's --prenorm line runs it: affinities, routing and the permuted
    e4m3 rows of the on-the-fly normalised x of all 64 tokens bit-exact
    against the oracle's pre-norm; every output row within tolerance."""
    from moe_inputs import make_residual
    cfg = CONFIGS["decode"]
    T, E, k, d = cfg.T, cfg.n_experts, cfg.top_k, cfg.d_model
    inp = make_inputs(cfg, seed=0, device=DEV)
    h, g = make_residual(cfg, seed=0, device=DEV)
    layer = moe.MoELayer(inp["w_router"], inp["bias"], inp["w13"], inp["w2"], top_k=k,
                         precision=cfg.precision)
    out = layer.forward_prenorm(h, g, 1e-6)
    assert layer.check_status(T) == 0
    off = moe.moe_workspace_layout(layer.shape(T))
    ws = layer.workspace(T)
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        ref = oracle.moe_layer_prenorm(
            u16(h), u16(g), 1e-6, u16(inp["w_router"]), inp["bias"].cpu().numpy(),
            lambda e: (u16(inp["w13"][e]), u16(inp["w2"][e])), n_experts=E,
            top_k=k, n_shared=cfg.n_shared, precision=cfg.precision, workers=min(WORKERS, 16))
    s = _ws_region(ws, off, "scores", T * E, torch.float32).reshape(T, E)
    assert np.array_equal(s.view(np.uint32), ref["scores"].view(np.uint32))
    assert np.array_equal(_ws_region(ws, off, "topk_idx", T * k, torch.int32).reshape(T, k),
                          ref["idx"])
    Rs = cfg.R_s
    a = _ws_region(ws, off, "a", Rs * d, torch.uint8).reshape(Rs, d)
    a_s = _ws_region(ws, off, "a_scales", Rs * (d // 128), torch.float32).reshape(Rs, d // 128)
    order = np.concatenate([ref["row_token"], np.arange(T, dtype=ref["row_token"].dtype)])
    assert np.array_equal(a, ref["xq"][order])
    assert np.array_equal(a_s.view(np.uint32), ref["xs"][order].view(np.uint32))
    assert_out_close(out, ref["out"], "prenorm decode", ref["out_allow"])
    del layer, inp
    torch.cuda.empty_cache()
