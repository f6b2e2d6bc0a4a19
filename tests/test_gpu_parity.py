"""GPU parity of every step of the layer against the oracle, through the C
ABI: routing (indices and gates bit-exact), permutation (bit-exact), e4m3
block quantisation (codes and scales bit-exact), grouped SwiGLU experts and
combine (tolerance), and the fused forward on the small workload, its ragged
and degenerate variants."""
import numpy as np
import pytest
import torch

import oracle
import sparse_moe_transformer_fwd_b200 as moe
from moe_inputs import CONFIGS, make_inputs

from _gpu_util import assert_close_to_correct, assert_out_close, from_u16, oracle_layer, u16, untile

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def _dev(inp):
    return {k: v.to(DEV) for k, v in inp.items()}


def _shape(cfg, **kw):
    c = cfg.with_(**kw) if kw else cfg
    return moe.make_shape(c.T, c.d_model, c.n_experts, c.top_k, c.d_expert, c.n_shared,
                          c.routed_scale, c.precision)


# ------------------------------------------------------------------ router --

ROUTE_CASES = {
    "tiny": CONFIGS["tiny"],
    "tiny_T1": CONFIGS["tiny"].with_(T=1),
    "tiny_T3": CONFIGS["tiny"].with_(T=3),
    "tiny_T127": CONFIGS["tiny"].with_(T=127),
    "tiny_T129": CONFIGS["tiny"].with_(T=129),
    "tiny_T600_bigtile": CONFIGS["tiny"].with_(T=600),
    "tiny_k16": CONFIGS["tiny"].with_(top_k=16),
    "tiny_scale2.5": CONFIGS["tiny"].with_(routed_scale=2.5),
    "decode": CONFIGS["decode"],
    "ds_T600_bigtile": CONFIGS["decode"].with_(T=600),
    # 64-token tiles launched with 2, 3 and 4 CTAs per SM at most (the
    # residency cap of launches that fit in one wave on 148 SMs)
    "tiny_T12000_cap2": CONFIGS["tiny"].with_(T=12000),
    "tiny_T24000_cap3": CONFIGS["tiny"].with_(T=24000),
    "tiny_T32000_cap4": CONFIGS["tiny"].with_(T=32000),
}


@pytest.mark.parametrize("name", list(ROUTE_CASES))
def test_route_bitexact(name):
    cfg = ROUTE_CASES[name]
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(cfg.T, cfg.d_model, generator=g)).to(torch.bfloat16)
    w = (torch.randn(cfg.n_experts, cfg.d_model, generator=g) * cfg.wr_std).to(torch.bfloat16)
    b = (torch.rand(cfg.n_experts, generator=g) * 0.2 - 0.1).float()
    shape = _shape(cfg)
    ws = moe.alloc_workspace(shape, DEV)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=DEV)
    gates = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=DEV)
    moe.moe_route(shape, x.to(DEV), w.to(DEV), b.to(DEV), idx, gates, ws)
    assert moe.moe_check_status(ws) == 0
    logits = oracle.router_logits(u16(x), u16(w))
    ridx, rg, _ = oracle.route(logits, b.numpy(), cfg.top_k, cfg.routed_scale)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.array_equal(gates.cpu().numpy().view(np.uint32), rg.view(np.uint32))


def test_route_ties_lowest_index():
    """All-zero router weights: every affinity is sigmoid(0) = 0.5, the bias
    decides, and equal biases go to the lowest expert index."""
    cfg = CONFIGS["tiny"].with_(T=40)
    x = torch.randn(cfg.T, cfg.d_model).to(torch.bfloat16)
    w = torch.zeros(cfg.n_experts, cfg.d_model, dtype=torch.bfloat16)
    b = torch.tensor([0.0, 0.1, 0.0, 0.1] * 4, dtype=torch.float32)
    shape = _shape(cfg)
    ws = moe.alloc_workspace(shape, DEV)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=DEV)
    gates = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=DEV)
    moe.moe_route(shape, x.to(DEV), w.to(DEV), b.to(DEV), idx, gates, ws)
    assert (idx.cpu() == torch.tensor([1, 3, 5, 7], dtype=torch.int32)).all()
    assert (gates.cpu() == 0.25).all()


# ------------------------------------------------------------- permutation --

def _rand_idx(rng, T, E, k, mode="uniform"):
    if mode == "uniform":
        return np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    if mode == "one":        # every token picks experts 0..k-1 (others empty)
        return np.tile(np.arange(k, dtype=np.int32), (T, 1))
    if mode == "skew":       # Zipf-like popularity
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        p /= p.sum()
        return np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    raise ValueError(mode)


PERM_CASES = [(1, 16, 4, "uniform"), (3, 16, 4, "uniform"), (257, 16, 4, "uniform"),
              (1000, 256, 8, "uniform"), (1000, 256, 8, "one"), (4096, 256, 8, "skew"),
              (600, 1023, 32, "uniform"), (64, 8, 8, "uniform"),
              # one 256-token block: the single-CTA path, up to its limits
              (256, 1023, 32, "uniform"), (256, 256, 8, "skew"), (255, 16, 16, "one")]


@pytest.mark.parametrize("T,E,k,mode", PERM_CASES)
def test_permute_bitexact(T, E, k, mode):
    rng = np.random.default_rng(T * 7 + E)
    idx = _rand_idx(rng, T, E, k, mode)
    shape = moe.make_shape(T, 256, E, k, 128, 1, 1.0, "fp8")
    ws = moe.alloc_workspace(shape, DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    row_token = torch.empty(T * k, dtype=torch.int32, device=DEV)
    row_of = torch.empty(T, k, dtype=torch.int32, device=DEV)
    moe.moe_permute(shape, torch.from_numpy(idx).to(DEV), counts, offsets, row_token, row_of, ws)
    assert moe.moe_check_status(ws) == 0
    rc, ro, rt, rr = oracle.permute(idx, E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(row_token.cpu().numpy(), rt)
    assert np.array_equal(row_of.cpu().numpy(), rr)


@pytest.mark.parametrize("T", [300, 250])
def test_permute_bad_index_reports_status(T):
    E, k = 16, 4
    rng = np.random.default_rng(5)
    idx = _rand_idx(rng, T, E, k)
    idx[7, 2] = E + 5          # out of range
    idx[200, 1] = idx[200, 0]  # duplicate within a token
    shape = moe.make_shape(T, 256, E, k, 128, 1, 1.0, "fp8")
    ws = moe.alloc_workspace(shape, DEV)
    outs = [torch.empty(n, dtype=torch.int32, device=DEV) for n in (E, E + 1, T * k, T * k)]
    moe.moe_permute(shape, torch.from_numpy(idx).to(DEV), *outs, ws)
    assert moe.moe_check_status(ws) == moe._native.MOE_ERR_DEVICE_INDEX
    assert moe.moe_check_status(ws) == 0   # cleared; the context is still usable
    torch.cuda.synchronize()


# ------------------------------------------------------------ quantisation --

QUANT_CASES = [(1, 128, 1), (1000, 7168, 1), (33, 384, 1), (256, 512, 128), (300, 384, 128),
               (4096, 7168, 128), (129, 128, 128)]


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("rows,cols,block_rows", QUANT_CASES)
def test_block_quant_bitexact(rows, cols, block_rows, ue8m0):
    g = torch.Generator().manual_seed(rows + cols)
    scale = torch.exp(torch.rand(rows, 1, generator=g) * 12 - 8)
    a = (torch.randn(rows, cols, generator=g) * scale).to(torch.bfloat16)
    a[0, :128] = 0.0                          # an all-zero tile
    if rows > 2:
        a[2, 5] = -0.0
        a[2, 130 % cols] = 1e30 if cols > 130 else a[2, 130 % cols]
    if ue8m0 and rows > 4:
        a[3, :128] *= 2.0 ** -120             # below the exponent floor 448 * 2^-128
        a[4, :128] = 0.0
        a[4, 1] = 448.0 * 2.0 ** -5           # amax exactly 448 * 2^j: scale 2^j
    q = torch.empty(rows, cols, dtype=torch.uint8, device=DEV)
    nrb = (rows + block_rows - 1) // block_rows
    s = torch.empty(nrb, cols // 128, dtype=torch.float32, device=DEV)
    moe.fp8_block_quant(a.to(DEV), block_rows, q, s, ue8m0=ue8m0)
    rq, rs = oracle.block_quant(u16(a), block_rows, ue8m0=ue8m0)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), rq)
    if block_rows == 128 and rows % 128 == 0:
        # tiled output: the same codes and scales, 128 x 128 tiles contiguous
        qt = torch.empty_like(q)
        st = torch.empty_like(s)
        moe.fp8_block_quant(a.to(DEV), block_rows, qt, st, layout=moe.MOE_LAYOUT_TILED,
                            ue8m0=ue8m0)
        assert torch.equal(st, s)
        assert np.array_equal(untile(qt.cpu().numpy(), rows, cols), rq)


@pytest.mark.parametrize("rows,row_bytes,dtype", [(128, 256, torch.bfloat16), (384, 1024, torch.uint8)])
def test_pack_tiles_is_the_tiled_permutation(rows, row_bytes, dtype):
    es = 2 if dtype == torch.bfloat16 else 1
    src = torch.randint(0, 255, (rows, row_bytes), dtype=torch.uint8).view(dtype)
    dst = torch.empty_like(src, device=DEV)
    moe.moe_pack_tiles(src.to(DEV), dst)
    got = untile(dst.cpu().contiguous().view(torch.uint8).numpy(), rows, row_bytes)
    assert np.array_equal(got, src.contiguous().view(torch.uint8).numpy().reshape(rows, row_bytes))


# ------------------------------------------- grouped experts and combine ---

@pytest.mark.parametrize("precision", ["bf16", "fp8", "fp8_ue8m0"])
@pytest.mark.parametrize("T", [128, 37])
def test_grouped_swiglu_and_combine(precision, T):
    cfg = CONFIGS["tiny"].with_(precision=precision, T=T)
    inp = make_inputs(cfg, seed=21)
    E, k = cfg.n_experts, cfg.top_k
    ref = oracle_layer(cfg, inp)
    # permuted activations built by the oracle
    rows = np.concatenate([ref["row_token"], np.arange(T)])
    shape = _shape(cfg)
    ws = moe.alloc_workspace(shape, DEV)
    y = torch.empty(cfg.R_s, cfg.d_model, dtype=torch.bfloat16, device=DEV)
    offsets = torch.from_numpy(ref["offsets"]).to(DEV)
    w13, w2 = inp["w13"].to(DEV), inp["w2"].to(DEV)
    ue = precision == "fp8_ue8m0"
    if precision != "bf16":
        a = torch.from_numpy(ref["xq"][rows]).to(DEV)
        a_s = torch.from_numpy(ref["xs"][rows]).to(DEV)
        w13q, w13s, w2q, w2s = moe.quantize_weights(w13, w2, ue8m0=ue)
        moe.moe_grouped_swiglu(shape, a, a_s, offsets, w13q, w13s, w2q, w2s, y, ws)
    else:
        a = from_u16(u16(inp["x"])[rows], DEV)
        w13t, w2t = moe.pack_weights(w13, w2)
        moe.moe_grouped_swiglu(shape, a, None, offsets, w13t, None, w2t, None, y, ws)
    assert moe.moe_check_status(ws) == 0
    # oracle expert outputs, row by row
    seg_of_row = np.concatenate([np.repeat(np.arange(E), ref["counts"]), np.full(T, E)])
    want = np.empty((cfg.R_s, cfg.d_model), np.uint16)
    want_allow = np.zeros((cfg.R_s, cfg.d_model))
    for e in range(E + 1):
        sel = np.nonzero(seg_of_row == e)[0]
        if sel.size == 0:
            continue
        w13e, w2e = u16(inp["w13"][e]), u16(inp["w2"][e])
        if precision != "bf16":
            q13, s13 = oracle.block_quant(w13e, 128, ue8m0=ue)
            q2, s2 = oracle.block_quant(w2e, 128, ue8m0=ue)
            want[sel], want_allow[sel] = oracle.expert_forward(
                ref["xq"][rows[sel]], q13, q2, precision, ref["xs"][rows[sel]], s13, s2,
                return_allow=True)
        else:
            want[sel] = oracle.expert_forward(u16(inp["x"])[rows[sel]], w13e, w2e, "bf16")
    assert_out_close(y, want, "grouped experts", want_allow)
    # combine
    out = torch.empty(T, cfg.d_model, dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(shape, y, torch.from_numpy(ref["row_of"]).to(DEV),
                    torch.from_numpy(ref["gates"]).to(DEV), out)
    yo = from_u16(want, DEV)
    out_ref = torch.empty_like(out)
    moe.moe_combine(shape, yo, torch.from_numpy(ref["row_of"]).to(DEV),
                    torch.from_numpy(ref["gates"]).to(DEV), out_ref)
    assert_out_close(out, ref["out"], "combine", ref["out_allow"])
    # combine alone, fed the oracle's Y: same as the oracle's combine
    assert_out_close(out_ref, ref["out"], "combine of oracle Y")


@pytest.mark.parametrize("precision", ["fp8", "bf16"])
def test_grouped_swiglu_long_caller_segments(precision):
    """Caller offsets with segments far longer than the batch: at T = 40 the
    fp32-scale GEMMs take 64-row tiles, so expert 0's 100 rows and expert 5's
    60 rows span several tiles (a 36-row ragged tile included)."""
    cfg = CONFIGS["tiny"].with_(precision=precision, T=40)
    inp = make_inputs(cfg, seed=22)
    E, k, T = cfg.n_experts, cfg.top_k, cfg.T
    R = T * k
    counts = np.zeros(E, np.int64)
    counts[0], counts[5] = 100, R - 100
    offsets_np = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = np.concatenate([(np.arange(R) * 7) % T, np.arange(T)])
    x16 = u16(inp["x"])
    shape = _shape(cfg)
    ws = moe.alloc_workspace(shape, DEV)
    y = torch.empty(cfg.R_s, cfg.d_model, dtype=torch.bfloat16, device=DEV)
    offsets = torch.from_numpy(offsets_np).to(DEV)
    w13, w2 = inp["w13"].to(DEV), inp["w2"].to(DEV)
    if precision == "fp8":
        xq, xs = oracle.block_quant(x16, 1)
        w13q, w13s, w2q, w2s = moe.quantize_weights(w13, w2)
        moe.moe_grouped_swiglu(shape, torch.from_numpy(xq[rows]).to(DEV),
                               torch.from_numpy(xs[rows]).to(DEV), offsets, w13q, w13s, w2q,
                               w2s, y, ws)
    else:
        w13t, w2t = moe.pack_weights(w13, w2)
        moe.moe_grouped_swiglu(shape, from_u16(x16[rows], DEV), None, offsets, w13t, None, w2t,
                               None, y, ws)
    assert moe.moe_check_status(ws) == 0
    # the oracle's rows, with their other correct H codes (nearest correct output)
    seg_of_row = np.concatenate([np.repeat(np.arange(E), counts), np.full(T, E)])
    res = dict(out_f64=np.zeros((cfg.R_s, cfg.d_model)), out_allow=np.zeros((cfg.R_s, cfg.d_model)),
               out_alts=[None] * cfg.R_s)
    for e in (0, 5, E):
        sel = np.nonzero(seg_of_row == e)[0]
        w13e, w2e = u16(inp["w13"][e]), u16(inp["w2"][e])
        if precision == "fp8":
            q13, s13 = oracle.block_quant(w13e, 128)
            q2, s2 = oracle.block_quant(w2e, 128)
            Y, al, alts = oracle.expert_forward(xq[rows[sel]], q13, q2, "fp8", xs[rows[sel]], s13,
                                                s2, return_f64=True, return_alts=True)
        else:
            Y, al, alts = oracle.expert_forward(x16[rows[sel]], w13e, w2e, "bf16",
                                                return_f64=True, return_alts=True)
        res["out_f64"][sel] = Y
        res["out_allow"][sel] = al
        for i, r in enumerate(sel):
            res["out_alts"][r] = alts[i]
    assert_close_to_correct(y, res, f"grouped experts, long caller segments, {precision}")


# -------------------------------------------------------- fused forward ---

FWD_CASES = {
    "tiny": dict(),
    "tiny_T1": dict(T=1),
    "tiny_T3": dict(T=3),
    "tiny_T127": dict(T=127),
    "tiny_T129": dict(T=129),
    "tiny_T600": dict(T=600),
    "tiny_noshared": dict(n_shared=0),
    "tiny_k16": dict(top_k=16),
    "tiny_scale2.5": dict(routed_scale=2.5),
    "tiny_wide": dict(d_model=1024, d_expert=512, n_experts=64, top_k=6, T=300),
    # at most 64 tokens: 64-row MMA tiles in the fp8 GEMMs (full shared
    # segment; and an odd number of K blocks in the down GEMM, d_expert 384)
    "tiny_T64": dict(T=64),
    "tiny_T48_de384": dict(T=48, d_expert=384),
    "tiny_T64_noshared": dict(T=64, n_shared=0),
}


@pytest.mark.parametrize("precision", ["bf16", "fp8", "fp8_ue8m0"])
@pytest.mark.parametrize("name", list(FWD_CASES))
def test_forward_vs_oracle(name, precision):
    cfg = CONFIGS["tiny"].with_(precision=precision, **FWD_CASES[name])
    inp = make_inputs(cfg, seed=3)
    d = _dev(inp)
    layer = moe.MoELayer(d["w_router"], d["bias"], d["w13"], d["w2"], top_k=cfg.top_k,
                         n_shared=cfg.n_shared, routed_scale=cfg.routed_scale,
                         precision=precision)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=DEV)
    out = layer(d["x"], topk_idx_out=idx)
    assert layer.check_status(cfg.T) == 0, moe.moe_last_error()
    ref = oracle_layer(cfg, inp)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    assert_out_close(out, ref["out"], name, ref["out_allow"])
    # deterministic: a second run gives the same bits
    out2 = layer(d["x"])
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("precision", ["bf16", "fp8", "fp8_ue8m0"])
def test_forward_all_tokens_on_few_experts(precision):
    """A large bias on experts 0..k-1 sends every token there: the other
    segments are empty and four segments hold T rows each (several tiles)."""
    cfg = CONFIGS["tiny"].with_(precision=precision, T=300)
    inp = make_inputs(cfg, seed=8)
    inp["bias"] = torch.zeros(cfg.n_experts)
    inp["bias"][: cfg.top_k] = 5.0
    d = _dev(inp)
    layer = moe.MoELayer(d["w_router"], d["bias"], d["w13"], d["w2"], top_k=cfg.top_k,
                         precision=precision)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=DEV)
    out = layer(d["x"], topk_idx_out=idx)
    assert layer.check_status(cfg.T) == 0
    ref = oracle_layer(cfg, inp)
    assert (np.sort(ref["idx"], 1) == np.arange(cfg.top_k)).all()
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    assert_out_close(out, ref["out"], "few experts", ref["out_allow"])


@pytest.mark.parametrize("precision", ["bf16", "fp8", "fp8_ue8m0"])
@pytest.mark.parametrize("T", [200, 40])
def test_rowmajor_weights_match_tiled(precision, T):
    """Expert weights in the problem statement's row-major layout, declared so
    in the shape (weight_layout MOE_LAYOUT_ROWMAJOR), give the tiled layer's
    routing and output bit for bit: the codes and the arithmetic are the
    same, only the coordinates of the weights' TMA boxes differ.  T=40 runs
    64-row tiles (fp32 scales), T=200 128-row tiles.  The same for the dense
    layer (split-K down GEMM at T=40)."""
    cfg = CONFIGS["tiny"].with_(precision=precision, T=T)
    d = _dev(make_inputs(cfg, seed=5))
    kw = dict(top_k=cfg.top_k, n_shared=cfg.n_shared, precision=precision)
    lt = moe.MoELayer(d["w_router"], d["bias"], d["w13"], d["w2"], weight_layout="tiled", **kw)
    lr = moe.MoELayer(d["w_router"], d["bias"], d["w13"], d["w2"], weight_layout="rowmajor", **kw)
    assert lr.shape(T).weight_layout == moe.MOE_LAYOUT_ROWMAJOR
    it = torch.empty(T, cfg.top_k, dtype=torch.int32, device=DEV)
    ir = torch.empty_like(it)
    ot, orr = lt(d["x"], topk_idx_out=it), lr(d["x"], topk_idx_out=ir)
    assert lt.check_status(T) == 0 and lr.check_status(T) == 0, moe.moe_last_error()
    assert torch.equal(it, ir)
    assert torch.equal(ot.view(torch.int16), orr.view(torch.int16))
    if precision != "bf16":
        n13, dm = lr.w13.shape[1:]
        assert np.array_equal(untile(lt.w13[3].cpu().numpy(), n13, dm), lr.w13[3].cpu().numpy())
    from moe_inputs import DENSE_CONFIGS, make_dense_inputs
    dc = DENSE_CONFIGS["dense_tiny"].with_(T=T, precision=precision)
    di = {k: v.to(DEV) for k, v in make_dense_inputs(dc, seed=5).items()}
    dt = moe.DenseFFN(di["w13"], di["w2"], precision=precision, weight_layout="tiled")
    dr = moe.DenseFFN(di["w13"], di["w2"], precision=precision, weight_layout="rowmajor")
    a, b = dt(di["x"]), dr(di["x"])
    assert dt.check_status(T) == 0 and dr.check_status(T) == 0, moe.moe_last_error()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_forward_empty_batch():
    cfg = CONFIGS["tiny"]
    inp = _dev(make_inputs(cfg, seed=1))
    layer = moe.MoELayer(inp["w_router"], inp["bias"], inp["w13"], inp["w2"], top_k=cfg.top_k,
                         precision="fp8")
    x = torch.empty(0, cfg.d_model, dtype=torch.bfloat16, device=DEV)
    out = layer(x)
    assert out.shape == (0, cfg.d_model)
    assert moe.moe_last_launch_count() == 0


def test_bounded_wait_timeout_reports_status(monkeypatch):
    """A pipeline stage armed for bytes that never arrive: the waiting thread
    gives up after its cycle budget, the call reports MOE_ERR_TIMEOUT through
    the status word, and the context stays usable."""
    cfg = CONFIGS["tiny"].with_(precision="fp8")
    inp = make_inputs(cfg, seed=2)
    d = _dev(inp)
    layer = moe.MoELayer(d["w_router"], d["bias"], d["w13"], d["w2"], top_k=cfg.top_k,
                         precision="fp8")
    monkeypatch.setenv("MOE_FAULT_INJECT", "gemm_tx")
    layer(d["x"])
    monkeypatch.delenv("MOE_FAULT_INJECT")
    assert layer.check_status(cfg.T) == moe._native.MOE_ERR_TIMEOUT
    out = layer(d["x"])
    assert layer.check_status(cfg.T) == 0
    ref = oracle_layer(cfg, inp)
    assert_out_close(out, ref["out"], "after timeout", ref["out_allow"])


# ----------------------------------------------- pre-norm block (fused) ---

PRENORM_CASES = {
    "tiny_bf16": CONFIGS["tiny"],
    "tiny_fp8": CONFIGS["tiny"].with_(precision="fp8"),
    "tiny_fp8_T600": CONFIGS["tiny"].with_(precision="fp8", T=600),
    "tiny_bf16_T3": CONFIGS["tiny"].with_(T=3),
    "tiny_fp8_T40": CONFIGS["tiny"].with_(precision="fp8", T=40),        # 64-row tiles
    "tiny_ue8m0_T100": CONFIGS["tiny"].with_(precision="fp8_ue8m0", T=100),
}


@pytest.mark.parametrize("name", list(PRENORM_CASES))
def test_forward_prenorm_vs_oracle(name):
    """out = h + MoE(bf16(RMSNorm(h) * gamma)) with x never materialised:
    routing bit-exact against the oracle's pre-norm, output within tolerance."""
    from moe_inputs import make_residual
    cfg = PRENORM_CASES[name]
    inp = make_inputs(cfg, seed=12)
    h, g = make_residual(cfg, seed=12)
    d = _dev(inp)
    layer = moe.MoELayer(d["w_router"], d["bias"], d["w13"], d["w2"], top_k=cfg.top_k,
                         precision=cfg.precision)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=DEV)
    out = layer.forward_prenorm(h.to(DEV), g.to(DEV), 1e-6, topk_idx_out=idx)
    assert layer.check_status(cfg.T) == 0
    ref = oracle.moe_layer_prenorm(
        u16(h), u16(g), 1e-6, u16(inp["w_router"]), inp["bias"].numpy(),
        lambda e: (u16(inp["w13"][e]), u16(inp["w2"][e])), n_experts=cfg.n_experts,
        top_k=cfg.top_k, n_shared=cfg.n_shared, precision=cfg.precision)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    assert_out_close(out, ref["out"], "prenorm " + name, ref["out_allow"])


def test_prenorm_router_decode_dims_bitexact():
    """Decode-size routing on normalised-on-the-fly inputs (small-batch router
    kernel) and a 600-token batch (tiled router kernel), DeepSeek dims."""
    from moe_inputs import make_residual
    for T in (64, 600):
        cfg = CONFIGS["decode"].with_(T=T)
        h, g = make_residual(cfg, seed=13)
        from moe_inputs import make_router
        w, b = make_router(cfg, seed=13)
        x_ref, _ = oracle.rmsnorm(u16(h), u16(g), 1e-6)
        logits = oracle.router_logits(x_ref, u16(w))
        ridx, rg, _ = oracle.route(logits, b.numpy(), cfg.top_k)
        # zero experts of width 128: only the routing and the residual are compared
        w13 = torch.zeros(cfg.n_experts + 1, 256, cfg.d_model, dtype=torch.bfloat16, device=DEV)
        w2 = torch.zeros(cfg.n_experts + 1, cfg.d_model, 128, dtype=torch.bfloat16, device=DEV)
        layer = moe.MoELayer(w.to(DEV), b.to(DEV), w13, w2, top_k=cfg.top_k, precision="bf16")
        idx = torch.empty(T, cfg.top_k, dtype=torch.int32, device=DEV)
        out = layer.forward_prenorm(h.to(DEV), g.to(DEV), 1e-6, topk_idx_out=idx)
        assert layer.check_status(T) == 0
        assert np.array_equal(idx.cpu().numpy(), ridx)
        # zero experts: the block returns the residual stream unchanged
        assert torch.equal(out.cpu().view(torch.int16), h.view(torch.int16))


# ------------------------------------------------------ launch records ---

@pytest.mark.parametrize("T,prenorm,precision", [(64, False, "fp8"), (300, False, "fp8"),
                                                 (64, True, "fp8"), (64, False, "bf16")])
def test_launch_names_follow_the_path(T, prenorm, precision):
    """moe_last_launch_name lists the kernels of the last call in launch order:
    the single-CTA permutation up to 256 tokens, three kernels beyond."""
    from moe_inputs import make_residual
    cfg = CONFIGS["tiny"].with_(precision=precision, T=T)
    inp = _dev(make_inputs(cfg, seed=9))
    layer = moe.MoELayer(inp["w_router"], inp["bias"], inp["w13"], inp["w2"], top_k=cfg.top_k,
                         precision=precision)
    h, gamma = make_residual(cfg, seed=9, device=DEV)
    run = (lambda: layer.forward_prenorm(h, gamma)) if prenorm else (lambda: layer(inp["x"]))
    run()
    assert layer.check_status(T) == 0
    run()  # the record belongs to the last call on this thread
    names = moe.moe_last_launch_names()
    perm = ["perm_small"] if T <= 256 else ["perm_hist", "perm_scan", "perm_scatter"]
    scatter = "quant_scatter" if precision == "fp8" else "scatter_bf16"
    want = (["prenorm_rstd"] if prenorm else []) + ["router_scores", "router_topk"] + perm + \
        [scatter, "grouped_gemm_gate_up", "grouped_gemm_down", "combine"]
    assert names == want
    assert moe.moe_last_launch_count() == len(want)
