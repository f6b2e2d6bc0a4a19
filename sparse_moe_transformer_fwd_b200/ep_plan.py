"""Exchange plan of an expert-parallel MoE layer: host logic only.

The routed experts are split contiguously over G ranks (rank r owns experts
r*P .. r*P + P - 1, P = E / G); every rank routes and permutes its own tokens
(moe_route, moe_permute), so its routed rows are in global expert order and
the rows for rank r's experts form one contiguous block.  From every rank's
per-expert row counts this module derives, for one rank:

  dispatch  how many rows it sends to each owner, and from where;
  receive   how many rows it gets from each source, and where they land
            (source-major, each source's block in expert order);
  segments  the grouped-GEMM segments of the received rows: one per
            (source, local expert), with its weight slot (the local expert);
  return    for each source, the row of that source's permuted order where
            this rank's results begin, so results can be stored straight
            back (or the dispatch all-to-all run in reverse).

Only the counts are exchanged here (one all_gather, NCCL on GPUs or gloo on
the CPU).  The data path that uses the plan is the library's
moe_ep_dispatch (rows pushed into the owners' receive buffers),
moe_ep_grouped_swiglu (the grouped GEMM over (source, expert) segments, Y
stored back from the down GEMM's epilogue into the source's buffer) and
moe_combine; dispatch_blocks and gemm_segments turn a plan into their
arguments.
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = ["EPPlan", "ep_plan", "exchange_counts", "dispatch_blocks", "gemm_segments"]


@dataclasses.dataclass(frozen=True)
class EPPlan:
    world: int
    rank: int
    experts_per_rank: int
    send_rows: np.ndarray   # [G] rows this rank sends to owner r
    send_start: np.ndarray  # [G] first row (this rank's permuted order) of the block for r
    recv_rows: np.ndarray   # [G] rows this rank receives from source s
    recv_start: np.ndarray  # [G] first row of source s's block in the receive buffer
    seg_source: np.ndarray  # [G*P] source rank of segment i (source-major order)
    seg_slot: np.ndarray    # [G*P] weight slot (local expert) of segment i
    seg_start: np.ndarray   # [G*P] first receive-buffer row of segment i
    seg_rows: np.ndarray    # [G*P] rows of segment i
    return_base: np.ndarray  # [G] row of source s's permuted order where this rank's rows begin

    @property
    def total_recv(self) -> int:
        return int(self.recv_rows.sum())


def _exclusive(a: np.ndarray) -> np.ndarray:
    out = np.zeros_like(a)
    np.cumsum(a[:-1], out=out[1:])
    return out


def ep_plan(counts_all, rank: int) -> EPPlan:
    """counts_all: int [G, E], row counts per (source rank, global expert),
    each rank's moe_permute counts.  E must be a multiple of G."""
    c = np.asarray(counts_all, dtype=np.int64)
    if c.ndim != 2 or np.any(c < 0):
        raise ValueError("counts_all must be a non-negative [G, E] array")
    G, E = c.shape
    if not 0 <= rank < G:
        raise ValueError(f"rank {rank} out of range for {G} ranks")
    if E % G:
        raise ValueError(f"{E} experts do not split evenly over {G} ranks")
    P = E // G
    owner_blocks = c.reshape(G, G, P)  # [source, owner, local expert]
    # this rank as a source: one contiguous block per owner, in owner order
    send_rows = owner_blocks[rank].sum(axis=1)
    send_start = _exclusive(send_rows)
    # this rank as an owner: source-major blocks of its P experts
    mine = owner_blocks[:, rank, :]      # [source, local expert]
    recv_rows = mine.sum(axis=1)
    recv_start = _exclusive(recv_rows)
    seg_rows = mine.reshape(-1)
    seg_start = _exclusive(seg_rows)
    seg_source = np.repeat(np.arange(G), P)
    seg_slot = np.tile(np.arange(P), G)
    # where this rank's block starts in each source's permuted order
    return_base = owner_blocks[:, :rank, :].reshape(G, -1).sum(axis=1)
    return EPPlan(G, rank, P, send_rows, send_start, recv_rows, recv_start, seg_source,
                  seg_slot, seg_start, seg_rows, return_base)


def exchange_counts(counts_local, group=None):
    """All ranks' per-expert counts, [G, E] (torch.distributed all_gather;
    counts_local is this rank's [E] tensor on the group's device)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(counts_local) for _ in range(world)]
    dist.all_gather(parts, counts_local, group=group)
    return torch.stack(parts)


def dispatch_blocks(counts_all, source: int):
    """The moe_ep_dispatch blocks of one source rank: for every owner o with
    rows from it, (first row in the source's permuted order, rows, o, first
    row in o's receive buffer)."""
    c = np.asarray(counts_all, dtype=np.int64)
    G = c.shape[0]
    mine = ep_plan(c, source)
    out = []
    for o in range(G):
        if mine.send_rows[o] == 0:
            continue
        dst_row = ep_plan(c, o).recv_start[source]
        out.append((int(mine.send_start[o]), int(mine.send_rows[o]), o, int(dst_row)))
    return out


def gemm_segments(plan: EPPlan, order: str = "slot"):
    """Segments of the owner's grouped GEMM as int32 arrays (start, rows,
    slot, source, return row): one per (source, local expert), the return
    row being where the segment's first row sits in its source's permuted
    order (return_base of the source plus its offset inside the source's
    block).  order "slot" lists them weight slot major (an expert's segments
    from all sources one after the other, so its weights are read while
    they are in L2), "source" in buffer order.  Empty segments are left out
    (at least one segment is kept)."""
    start = plan.seg_start.astype(np.int64)
    src = plan.seg_source.astype(np.int64)
    ret = plan.return_base[src] + (start - plan.recv_start[src])
    keys = np.lexsort((src, plan.seg_slot)) if order == "slot" else np.arange(len(start))
    keep = [i for i in keys if plan.seg_rows[i] > 0] or [int(keys[0])]
    idx = np.array(keep, dtype=np.int64)
    i32 = lambda a: np.ascontiguousarray(a[idx], dtype=np.int32)
    return {"seg_start": i32(start), "seg_rows": i32(plan.seg_rows), "seg_slot": i32(plan.seg_slot),
            "seg_src": i32(src), "seg_ret": i32(ret)}
