"""The N>1 path of bench.py (independent replicas, one per rank) on CPU with
two gloo ranks: the barrier, the max-over-ranks step time and the whole-job
throughput.  The layer itself has no exchange step, so nothing else crosses
ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.dist_setup(world, backend="gloo")
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    local_ms = 1.0 + rank * 0.25            # rank 1 is the slower one
    ms = bench.max_over_ranks(local_ms, w, torch.device("cpu"))
    q.put((rank, ms, bench.job_throughput(64, w, ms)))
    bench.barrier(w)
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_max_and_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in res] == [0, 1]
    assert all(ms == pytest.approx(1.25) for _, ms, _ in res)          # max over ranks
    assert all(v == pytest.approx(128 / 1.25e-3) for _, _, v in res)   # 2 x 64 tokens / slowest


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    assert bench.job_throughput(64, 1, 2.0) == pytest.approx(32000.0)
