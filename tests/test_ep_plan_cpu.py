"""The exchange plan of an expert-parallel layer (host logic) on the CPU:
its invariants, a single-process simulation of dispatch and return that
follows every routed row, gloo ranks that exchange their counts and then move
routed-row ids through all-to-alls sized by the plan and back, and an
expert-parallel forward on four gloo ranks (the oracle as the compute) that
reproduces the data-parallel layer."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from sparse_moe_transformer_fwd_b200.ep_plan import ep_plan


def _idx(rng, T, E, k, skew=False):
    p = None
    if skew:
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        p /= p.sum()
    return np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def _row_ids(idx, E, source):
    """Permuted rows of one source rank (moe_permute's order: expert, then
    token) as ids source * 10^6 + expert * 10^3 + token."""
    counts, offsets, row_token, _ = oracle.permute(idx, E)
    expert = np.repeat(np.arange(E), counts)
    return source * 1_000_000 + expert * 1000 + row_token.astype(np.int64), counts


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("skew", [False, True])
def test_plan_invariants(G, skew):
    rng = np.random.default_rng(G * 10 + skew)
    E = 64
    counts = np.stack([np.bincount(_idx(rng, 50 + 9 * s, E, 4, skew).ravel(), minlength=E)
                       for s in range(G)])
    for r in range(G):
        p = ep_plan(counts, r)
        P = E // G
        assert p.send_rows.sum() == counts[r].sum()
        assert np.array_equal(p.send_rows, counts[r].reshape(G, P).sum(1))
        assert np.array_equal(p.recv_rows, counts[:, r * P:(r + 1) * P].sum(1))
        # the segments tile the receive buffer, source-major, expert order within
        assert p.seg_start[0] == 0
        assert np.array_equal(p.seg_start[1:], np.cumsum(p.seg_rows)[:-1])
        assert p.seg_rows.sum() == p.total_recv
        assert np.array_equal(p.seg_rows.reshape(G, P).sum(1), p.recv_rows)
        assert np.array_equal(p.seg_start.reshape(G, P)[:, 0], p.recv_start)
        assert np.array_equal(p.return_base, counts[:, :r * P].sum(1))
    if G == 1:  # one rank: its own segments, one per expert
        p = ep_plan(counts, 0)
        assert np.array_equal(p.seg_rows, counts[0])


def test_plan_rejects_bad_input():
    with pytest.raises(ValueError):
        ep_plan(np.zeros((3, 64)), 0)        # 64 experts over 3 ranks
    with pytest.raises(ValueError):
        ep_plan(np.zeros((2, 64)), 2)        # no such rank
    with pytest.raises(ValueError):
        ep_plan(-np.ones((2, 64)), 0)


def test_single_process_dispatch_and_return():
    """Every routed row of every source lands in its owner's segment for its
    expert (in token order), and the return rows give back the row's place
    in its source's permuted order."""
    rng = np.random.default_rng(5)
    G, E, k = 4, 32, 4
    P = E // G
    ids, counts = zip(*[_row_ids(_idx(rng, 40 + 7 * s, E, k), E, s) for s in range(G)])
    counts = np.stack(counts)
    plans = [ep_plan(counts, r) for r in range(G)]
    recv = []
    for r in range(G):
        blocks = [ids[s][plans[s].send_start[r]:plans[s].send_start[r] + plans[s].send_rows[r]]
                  for s in range(G)]
        recv.append(np.concatenate(blocks))
        assert len(recv[r]) == plans[r].total_recv
    for r, p in enumerate(plans):
        for i in range(G * P):
            rows = recv[r][p.seg_start[i]:p.seg_start[i] + p.seg_rows[i]]
            s, slot = p.seg_source[i], p.seg_slot[i]
            assert np.all(rows // 1_000_000 == s)
            assert np.all((rows // 1000) % 1000 == r * P + slot)
            assert np.all(np.diff(rows % 1000) > 0)            # tokens ascend
        for s in range(G):
            block = recv[r][p.recv_start[s]:p.recv_start[s] + p.recv_rows[s]]
            back = p.return_base[s] + np.arange(len(block))
            assert np.array_equal(ids[s][back], block)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    from sparse_moe_transformer_fwd_b200.ep_plan import exchange_counts
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        E, k = 16, 4
        P = E // world
        ids, counts = _row_ids(_idx(np.random.default_rng(100 + rank), 30 + 11 * rank, E, k), E, rank)
        counts_all = exchange_counts(torch.from_numpy(counts.astype(np.int64))).numpy()
        p = ep_plan(counts_all, rank)
        send = torch.from_numpy(ids)
        recv = torch.empty(p.total_recv, dtype=torch.int64)
        dist.all_to_all_single(recv, send, output_split_sizes=p.recv_rows.tolist(),
                               input_split_sizes=p.send_rows.tolist())
        r_np = recv.numpy()
        ok = True
        for i in range(world * P):
            rows = r_np[p.seg_start[i]:p.seg_start[i] + p.seg_rows[i]]
            ok &= bool(np.all(rows // 1_000_000 == p.seg_source[i]))
            ok &= bool(np.all((rows // 1000) % 1000 == rank * P + p.seg_slot[i]))
        # results go back the same way: the reverse all-to-all restores the
        # source's permuted order exactly
        back = torch.empty_like(send)
        dist.all_to_all_single(back, recv, output_split_sizes=p.send_rows.tolist(),
                               input_split_sizes=p.recv_rows.tolist())
        ok &= bool(torch.equal(back, send))
        q.put((rank, ok, int(p.total_recv)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_exchange_rows_by_the_plan(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in res] == list(range(world))
    assert all(ok for _, ok, _ in res)
    # every routed row of every rank was received by exactly one owner
    assert sum(n for _, _, n in res) == sum((30 + 11 * r) * 4 for r in range(world))


def _layer_worker(rank, world, port, q):
    """One rank of an expert-parallel forward with the oracle as compute:
    route and permute locally, dispatch rows by the plan, evaluate each
    (source, expert) segment with its slot's weights, return Y by the reverse
    all-to-all, combine; then the data-parallel oracle layer on the same
    tokens for comparison."""
    import torch.distributed as dist
    from moe_inputs import CONFIGS, make_inputs, make_x
    from sparse_moe_transformer_fwd_b200.ep_plan import exchange_counts
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        T = 24 + 5 * rank
        cfg = CONFIGS["tiny"].with_(T=T)
        inp = make_inputs(cfg, seed=7)               # the same weights on every rank
        x = make_x(cfg, seed=70 + rank)               # each rank its own tokens
        u = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
        E, k, d = cfg.n_experts, cfg.top_k, cfg.d_model
        P = E // world
        x16, wr = u(x), u(inp["w_router"])
        idx, gates, _ = oracle.route(oracle.router_logits(x16, wr), inp["bias"].numpy(), k)
        counts, offsets, row_token, row_of = oracle.permute(idx, E)
        p = ep_plan(exchange_counts(torch.from_numpy(counts.astype(np.int64))).numpy(), rank)
        # dispatch the routed rows (bf16 bits as int32 for the exchange)
        send = torch.from_numpy(x16[row_token].astype(np.int32))
        recv = torch.empty(p.total_recv, d, dtype=torch.int32)
        dist.all_to_all_single(recv, send, output_split_sizes=p.recv_rows.tolist(),
                               input_split_sizes=p.send_rows.tolist())
        rows = recv.numpy().astype(np.uint16)
        # each segment with its weight slot (local expert -> global expert)
        y = np.zeros((p.total_recv, d), dtype=np.uint16)
        for i in range(world * P):
            a, n = p.seg_start[i], p.seg_rows[i]
            if n:
                e = rank * P + p.seg_slot[i]
                y[a:a + n] = oracle.expert_forward(rows[a:a + n], u(inp["w13"][e]), u(inp["w2"][e]),
                                                   "bf16")
        back = torch.empty(int(p.send_rows.sum()), d, dtype=torch.int32)
        dist.all_to_all_single(back, torch.from_numpy(y.astype(np.int32)),
                               output_split_sizes=p.send_rows.tolist(),
                               input_split_sizes=p.recv_rows.tolist())
        yr = oracle.bf16_to_f32(back.numpy().astype(np.uint16)).astype(np.float64)
        ys = oracle.bf16_to_f32(oracle.expert_forward(x16, u(inp["w13"][E]), u(inp["w2"][E]),
                                                      "bf16")).astype(np.float64)
        acc = np.einsum("tj,tjd->td", gates.astype(np.float64), yr[row_of]) + ys
        out_ep = oracle.bf16_from_f32(acc.astype(np.float32))
        ref = oracle.moe_layer(x16, wr, inp["bias"].numpy(),
                               lambda e: (u(inp["w13"][e]), u(inp["w2"][e])), n_experts=E,
                               top_k=k, n_shared=1, precision="bf16")["out"]
        a64 = oracle.bf16_to_f32(out_ep).astype(np.float64)
        b64 = oracle.bf16_to_f32(ref).astype(np.float64)
        step = np.abs(b64) * 2.0 ** -7 + 1e-30
        q.put((rank, bool(np.all(np.abs(a64 - b64) <= step)), float((out_ep != ref).mean())))
    finally:
        dist.destroy_process_group()


def test_gloo_expert_parallel_forward_matches_the_layer():
    world, port = 4, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_layer_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in res] == list(range(world))
    # the expert outputs are the same binary64 products evaluated in other
    # row batches: within one bf16 step, almost every bit equal
    assert all(ok for _, ok, _ in res)
    assert all(frac < 0.01 for _, _, frac in res)


@pytest.mark.parametrize("G", [1, 2, 4])
def test_dispatch_blocks_and_gemm_segments_follow_every_row(G):
    """dispatch_blocks and gemm_segments, the arguments of moe_ep_dispatch and
    moe_ep_grouped_swiglu: every routed row of every source is sent once,
    lands in its owner's receive buffer inside exactly one segment whose slot
    is its expert, and returns to the row it came from in its source's
    permuted order."""
    from sparse_moe_transformer_fwd_b200.ep_plan import dispatch_blocks, gemm_segments
    rng = np.random.default_rng(40 + G)
    E, k = 16, 4
    idxs = [_idx(rng, 20 + 13 * s, E, k, skew=bool(s % 2)) for s in range(G)]
    perm = [_row_ids(idx, E, s) for s, idx in enumerate(idxs)]
    counts = np.stack([c for _, c in perm])
    P = E // G
    recv = [np.full(ep_plan(counts, o).total_recv, -1, dtype=np.int64) for o in range(G)]
    for s in range(G):
        ids = perm[s][0]
        for src_row, rows, o, dst_row in dispatch_blocks(counts, s):
            assert np.all(recv[o][dst_row:dst_row + rows] == -1)      # no overlap
            recv[o][dst_row:dst_row + rows] = ids[src_row:src_row + rows]
    returned = [np.full(len(perm[s][0]), -1, dtype=np.int64) for s in range(G)]
    for o in range(G):
        assert np.all(recv[o] >= 0)                                  # every row filled
        segs = gemm_segments(ep_plan(counts, o))
        covered = np.zeros(len(recv[o]), dtype=int)
        for st, n, slot, src, ret in zip(*(segs[k] for k in ("seg_start", "seg_rows", "seg_slot",
                                                                 "seg_src", "seg_ret"))):
            rows = recv[o][st:st + n]
            covered[st:st + n] += 1
            assert np.all(rows // 1_000_000 == src)                   # from that source
            assert np.all((rows // 1000) % 1000 == o * P + slot)      # of that expert
            returned[src][ret:ret + n] = rows
        assert np.all(covered == 1)
        # weight-slot-major order
        assert np.all(np.diff(segs["seg_slot"]) >= 0)
    for s in range(G):
        assert np.array_equal(returned[s], perm[s][0])                # back where it came from
