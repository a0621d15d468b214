"""Data-parallel replicas: one process per GPU, each decoding its own batch.

Every (sequence, KV head) of a decode step is independent through metadata, scoring, selection
and attention, so the path shards by batch with no collective on the data path. The only
cross-rank steps are the timing ones: a barrier around the timed region and the maximum of the
ranks' device-timed intervals (the whole job is as fast as its slowest rank).
"""
from __future__ import annotations

import os

import torch

WORKLOAD_SEEDS = {"tiny": 1, "gqa32k": 2, "needle128k": 3, "gauss": 4, "long1m": 5}


def rank_info():
    """(rank, world_size, local_rank) from the launcher's environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def workload_seed(name: str, rank: int) -> int:
    """Each rank decodes its own seeded batch."""
    return WORKLOAD_SEEDS[name] + 1000 * rank


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest `value` over all ranks (identity without an initialised process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def job_rate(steps_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job steps per second: every rank ran `steps_per_rank` steps of its own batch."""
    return world * steps_per_rank / max_seconds
