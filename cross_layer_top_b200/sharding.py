"""Prefill split across ranks: the plumbing around ic_run_stack_rows.

The prefill path splits by query rows.  Given the whole k_I, K and V, a query
row's scores, top-k and attention need nothing from another row (the
reading-notes page, §2.1 and §3).  So each rank
  1. takes its rows from ic_prefill_partition, a causal-balanced (zig-zag)
     split in which rank r owns chunks r and 2W-1-r of 2W near-equal chunks;
  2. holds its own rows of every layer's tensors (it produced them);
  3. all-gathers its rows of k_I, K and V (one collective per tensor, NCCL
     over NVLink on GPUs, gloo on CPU), then runs ic_run_stack_rows locally.

This module only moves data.  The partition and every computation live in
libindexcache.so.  The gathered rows are placed at their positions with
plain tensor copies.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import indexcache as ic


def partition(L: int, world: int):
    """Row ranges of every rank: [[(a0, b0), (a1, b1)] for rank 0, ...]."""
    return [ic.ic_prefill_partition(L, world, r) for r in range(world)]


def rows_of(full: torch.Tensor, ranges) -> torch.Tensor:
    """The rows of `full` in `ranges`, range after range (a rank's share of a
    tensor drawn whole, e.g. synthetic inputs with a shared seed)."""
    return torch.cat([full[a:b] for a, b in ranges]).contiguous()


def allgather_rows(local: torch.Tensor, ranges_all, L: int, group=None) -> torch.Tensor:
    """Every rank's rows of a [L, ...] tensor, put back in position order.

    local: this rank's rows (ranges_all[rank], range after range).  All ranks
    call this with the same ranges_all, in the same order.  Returns the whole
    [L, ...] tensor on local's device."""
    if len(ranges_all) == 1:  # one rank: its rows are every row, in order
        full = local.new_empty((L,) + tuple(local.shape[1:]))
        off = 0
        for a, b in ranges_all[0]:
            full[a:b] = local[off:off + b - a]
            off += b - a
        return full
    counts = [sum(b - a for a, b in rr) for rr in ranges_all]
    cmax = max(counts)
    send = local
    if local.shape[0] < cmax:  # equal-size buffers for the collective
        pad = local.new_zeros((cmax - local.shape[0],) + tuple(local.shape[1:]))
        send = torch.cat([local, pad])
    bufs = [torch.empty_like(send) for _ in ranges_all]
    dist.all_gather(bufs, send.contiguous(), group=group)
    full = local.new_empty((L,) + tuple(local.shape[1:]))
    for r, rr in enumerate(ranges_all):
        off = 0
        for a, b in rr:
            full[a:b] = bufs[r][off:off + b - a]
            off += b - a
    return full
