"""One process per GPU, independent sequences per rank (weak scaling).

PIVOT indexes each sequence's groups independently of every other sequence,
so N GPUs index N sequences with no collective on the data path; the only
collectives are the barriers around a timed region and one max-reduction of
the per-rank time.  The whole-job throughput is the queries of all ranks over
the slowest rank's time.
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch
import torch.distributed as dist

SEED_STRIDE = 7919  # rank r draws its sequence from seed + SEED_STRIDE * r


def env() -> Tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment (1, 0, 0 when absent)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, world: int, timeout_s: float = 300.0) -> None:
    """Join the process group when world > 1 (env:// rendezvous; MASTER_ADDR must be set)."""
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s sequence: rank 0 keeps the workload's own seed."""
    return seed + SEED_STRIDE * rank


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The maximum of x over all ranks (x itself when world == 1)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling(total_ms_local: float, steps: int, units_per_rank: int, world: int, device=None):
    """(ms per step, whole-job units/s): every rank processed units_per_rank per step;
    the job takes as long as its slowest rank."""
    total_ms = max_over_ranks(total_ms_local, world, device)
    ms = total_ms / steps
    return ms, world * units_per_rank / (ms / 1000.0)


def finish(world: int) -> None:
    """Every rank calls this last: a final barrier, then leave the process group."""
    if world > 1 and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


__all__ = ["SEED_STRIDE", "env", "init", "rank_seed", "barrier", "max_over_ranks", "weak_scaling", "finish"]
