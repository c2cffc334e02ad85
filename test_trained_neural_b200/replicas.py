"""One process per GPU: every rank runs its own replica of a workload.

Streams (batch entry, head) of the memory are independent, so a multi-GPU run
needs no exchange on the data path: rank r runs the whole workload with its
own seed, and only the timing is combined (max over ranks) with one
collective. Throughput = ranks x tokens per replica / max time.
"""
from __future__ import annotations

import dataclasses

RANK_SEED_STRIDE = 1000


def replica(w, rank: int):
    """The workload `w` as drawn by rank `rank` (rank 0 is `w` itself)."""
    if rank == 0:
        return w
    return dataclasses.replace(w, index=w.index + RANK_SEED_STRIDE * rank)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity for one rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(tokens_per_replica: int, world: int, max_seconds: float) -> float:
    return world * tokens_per_replica / max_seconds
