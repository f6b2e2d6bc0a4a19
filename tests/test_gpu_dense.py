"""GPU parity of the dense gated FFN layer (the model's first layers,
"DeepSeek-R1" card, "Every architecture field": ffns.dense gated, d_ff 18432)
against the oracle, through the C ABI.

Small shapes cover the down GEMM's split K (even and uneven K ranges, 64- and
128-row tiles, bf16), the single-range path past 256 tokens, UE8M0 block
scales, the pre-norm block with the residual fused into the down GEMM, T = 0,
the launch record, and bit-identical repeats (the split-K sum has a fixed
order).  The DeepSeek-V3 dense layer runs
at the decode and prefill batches, compared on sampled rows."""
import numpy as np
import pytest
import torch

import oracle
import sparse_moe_transformer_fwd_b200 as moe
from moe_inputs import DENSE_CONFIGS, make_dense_inputs, make_residual

from _gpu_util import assert_close_to_correct, u16, untile

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None
TINY = DENSE_CONFIGS["dense_tiny"]

# (config, what the down GEMM does at 148 SMs)
CASES = {
    "T100_ff768": TINY,                                          # split 3, ranges of 2
    "T48_ff640": TINY.with_(T=48, d_ff=640),                     # 64-row tiles, split 2 (2 + 3)
    "T64_d1024_ff1152": TINY.with_(T=64, d_model=1024, d_ff=1152),  # split 4 (2,2,2,3)
    "T300": TINY.with_(T=300),                                   # 3 row tiles, no split
    "T1": TINY.with_(T=1),
    "T257": TINY.with_(T=257),                                   # first batch without split
    "bf16_T100": TINY.with_(precision="bf16"),                   # split over 64-wide K blocks
    "ue8m0_T100": TINY.with_(precision="fp8_ue8m0"),             # block-scaled MMA, no split
}


def _layer(cfg, seed):
    inp = {k: v.to(DEV) for k, v in make_dense_inputs(cfg, seed=seed).items()}
    return inp, moe.DenseFFN(inp["w13"], inp["w2"], precision=cfg.precision)


def _oracle(cfg, inp, tokens=None):
    return oracle.dense_ffn(u16(inp["x"]), u16(inp["w13"]), u16(inp["w2"]),
                            precision=cfg.precision, tokens=tokens)


@pytest.mark.parametrize("name", list(CASES))
def test_dense_vs_oracle(name):
    cfg = CASES[name]
    inp, layer = _layer(cfg, seed=21)
    out = layer(inp["x"])
    assert layer.check_status(cfg.T) == 0
    res = _oracle(cfg, inp)
    assert_close_to_correct(out, res, f"dense {name}")


@pytest.mark.parametrize("precision", ["fp8", "fp8_ue8m0"])
def test_dense_weight_codes_bitexact(precision):
    cfg = TINY.with_(precision=precision)
    inp, layer = _layer(cfg, seed=22)
    ue = precision == "fp8_ue8m0"
    for w, q, s in ((inp["w13"], layer.w13, layer.w13s), (inp["w2"], layer.w2, layer.w2s)):
        rq, rs = oracle.block_quant(u16(w), 128, ue8m0=ue)
        got = untile(q.cpu().numpy(), w.shape[0], w.shape[1])
        assert np.array_equal(got, rq)
        assert np.array_equal(s.cpu().numpy().reshape(rs.shape), rs)


@pytest.mark.parametrize("name,precision", [("T48", "fp8"), ("T300", "fp8"), ("T100", "bf16"),
                                            ("T64", "fp8_ue8m0")])
def test_dense_prenorm_vs_oracle(name, precision):
    T = int(name[1:])
    cfg = TINY.with_(T=T, precision=precision)
    inp, layer = _layer(cfg, seed=23)
    h, gamma = make_residual(cfg, seed=23, device=DEV)
    out = layer.forward_prenorm(h, gamma, 1e-6)
    assert layer.check_status(T) == 0
    res = oracle.dense_ffn_prenorm(u16(h), u16(gamma), 1e-6, u16(inp["w13"]), u16(inp["w2"]),
                                   precision=precision)
    assert_close_to_correct(out, res, f"dense prenorm {name} {precision}")


@pytest.mark.parametrize("name", ["T48_ff640", "T100_ff768", "bf16_T100"])
def test_dense_split_k_repeats_bitidentical(name):
    """Three calls give identical bits: the K ranges' partial sums are added
    in K order, whatever order the blocks ran in."""
    cfg = CASES[name]
    inp, layer = _layer(cfg, seed=24)
    outs = [layer(inp["x"]).clone() for _ in range(3)]
    assert layer.check_status(cfg.T) == 0
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))


def test_dense_empty_batch():
    cfg = TINY.with_(T=0)
    inp, layer = _layer(TINY, seed=25)
    out = torch.empty(0, cfg.d_model, dtype=torch.bfloat16, device=DEV)
    layer(inp["x"][:0], out=out)
    assert moe.moe_last_launch_count() == 0


@pytest.mark.parametrize("precision,prenorm", [("fp8", False), ("fp8", True), ("bf16", False),
                                               ("bf16", True)])
def test_dense_launch_names(precision, prenorm):
    cfg = TINY.with_(precision=precision)
    inp, layer = _layer(cfg, seed=26)
    h, gamma = make_residual(cfg, seed=26, device=DEV)
    (layer.forward_prenorm(h, gamma) if prenorm else layer(inp["x"]))
    names = moe.moe_last_launch_names()
    first = (["prenorm_rstd"] if prenorm else []) + \
        (["quant_scatter"] if precision == "fp8" else (["scatter_bf16"] if prenorm else []))
    # 100 tokens: the down GEMM splits K, and a reduce kernel adds the ranges
    assert names == first + ["grouped_gemm_gate_up", "grouped_gemm_down", "splitk_reduce"]
    # past 256 tokens, no split: the down GEMM stores out (and adds h) itself
    big = TINY.with_(T=300, precision=precision)
    inp, layer = _layer(big, seed=26)
    h, gamma = make_residual(big, seed=26, device=DEV)
    (layer.forward_prenorm(h, gamma) if prenorm else layer(inp["x"]))
    assert moe.moe_last_launch_names() == first + ["grouped_gemm_gate_up", "grouped_gemm_down"]


def test_dense_rejects_bad_shapes():
    x = torch.zeros(4, 512, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(moe.MoeError):
        moe.moe_dense_workspace_size(moe.make_dense_shape(4, 384, 768))
    with pytest.raises(moe.MoeError):
        moe.moe_dense_workspace_size(moe.make_dense_shape(4, 512, 700))
    shape = moe.make_dense_shape(4, 512, 768)
    ws = moe.alloc_dense_workspace(shape, DEV)
    out = torch.empty_like(x)
    w13 = torch.zeros(1536, 512, dtype=torch.uint8, device=DEV)
    w2 = torch.zeros(512, 768, dtype=torch.uint8, device=DEV)
    s13 = torch.ones(12, 4, device=DEV)
    s2 = torch.ones(4, 6, device=DEV)
    with pytest.raises(moe.MoeError):  # workspace too small
        moe.moe_dense_ffn(shape, x, w13, s13, w2, s2, out, ws[:1024])
    with pytest.raises(moe.MoeError):  # fp8 needs scales
        moe.moe_dense_ffn(shape, x, w13, None, w2, s2, out, ws)


# ------------------------------------------------- DeepSeek-V3 dense layer --

@pytest.mark.parametrize("name,n_sample", [("dense_decode", 8), ("dense_prefill", 6)])
def test_dense_fullsize_sampled(name, n_sample):
    cfg = DENSE_CONFIGS[name]
    inp, layer = _layer(cfg, seed=0)
    out = layer(inp["x"])
    assert layer.check_status(cfg.T) == 0
    rng = np.random.default_rng(3)
    tok = np.sort(rng.choice(cfg.T, n_sample, replace=False))
    tok[-1] = cfg.T - 1  # the ragged last row tile
    res = _oracle(cfg, {k: v.cpu() for k, v in inp.items()}, tokens=tok)
    assert_close_to_correct(out[torch.as_tensor(tok, device=DEV)], res, f"{name} sampled")
