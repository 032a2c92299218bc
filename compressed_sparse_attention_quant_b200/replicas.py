"""Host logic of the multi-GPU run: one independent replica per rank.

The decode path shards by sequence with no exchange step, so N GPUs run N
replicas of the same per-rank batch (weak scaling) and the only collective
is the reduction of the timing scalars, outside the timed region:
  * rank r draws its inputs from seed + 1000 * r (independent replicas);
  * every rank measures on its own device; the job time of a step is the
    maximum over ranks;
  * whole-job throughput = tokens of all ranks / that maximum;
  * rank 0 alone reports.
"""
from __future__ import annotations

import dataclasses
from typing import Sequence

import torch

from .inputs import Workload

SEED_STRIDE = 1000


def replica_workload(wl: Workload, rank: int) -> Workload:
    """The workload rank `rank` runs: same shapes, its own seed."""
    return dataclasses.replace(wl, seed=wl.seed + SEED_STRIDE * rank) if rank else wl


def max_over_ranks(values: Sequence[float], dist=None, device=None) -> list:
    """Element-wise maximum of per-rank timing scalars (identity on one rank)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(tokens_per_rank: int, world: int, step_ms: float) -> float:
    """Whole-job tokens per second over all ranks."""
    return tokens_per_rank * world / (step_ms * 1e-3)


def reports(rank: int) -> bool:
    """Only rank 0 prints the result line."""
    return rank == 0
