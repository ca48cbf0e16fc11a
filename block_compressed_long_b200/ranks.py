"""One process per GPU: rank layout, per-rank workloads and the reduction of
device-timed results over ranks.

Decode is independent per sequence (and per kv head), so the ranks of a
multi-GPU run decode disjoint sequences and exchange nothing on the data path:
weak scaling, with the step time of the job the slowest rank's.  The only
collectives are the barriers around the timed region and the max of the
timings.  Host logic only; it works with any torch.distributed backend (NCCL
between GPUs, gloo on CPU).
"""
from __future__ import annotations

import os
from dataclasses import replace

import torch
import torch.distributed as dist

# odd stride between the seeds of consecutive ranks: every rank draws its own
# sequences from the same workload recipe
RANK_SEED_STRIDE = 7919


def from_env() -> tuple[int, int, int]:
    """(rank, world size, local rank) as torch.distributed.run exports them;
    (0, 1, 0) for a plain single-process run."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_workload(w, rank: int):
    """The workload a rank runs under weak scaling: the same shapes and length
    mix, its own seeded sequences."""
    return replace(w, seed=w.seed + RANK_SEED_STRIDE * rank)


def shard_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [lo, hi) share of n independent units (sequences) for a rank
    when a fixed global batch is split (strong scaling); sizes differ by at
    most one and every unit has exactly one owner."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    q, r = divmod(n, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def max_over_ranks(values, device=None) -> list[float]:
    """Element-wise max over all ranks of a list of floats (a no-op without an
    initialised process group).  Every rank must call it, in the same order."""
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def job_us_per_token(step_ms: float, tokens_per_rank: int, world: int) -> float:
    """Whole-job decode time per token: the (max over ranks) step time over the
    tokens that all ranks decoded in that step."""
    return step_ms * 1e3 / (tokens_per_rank * world)
