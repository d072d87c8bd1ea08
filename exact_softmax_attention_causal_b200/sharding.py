"""Host-side logic for running the hot path on several GPUs at once.

The work partitions into independent units (a prefill's (batch, head, query
tile) items, a decode's (sequence, K/V head) pairs), so N GPUs need no
collective on the data path: every rank processes its own units. Two ways to
hand them out:

* weak scaling (what the benchmark does): every rank runs a full batch of its
  own, drawn from a rank-specific seed;
* strong scaling of one global batch: contiguous, near-equal slices of the
  batch dimension, one per rank.

The only communication is for timing: the step time is the maximum over
ranks (an all-reduce of a few floats), and throughput counts all ranks' work.
"""

from __future__ import annotations

import torch


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s independent batch (rank 0 keeps `seed`)."""
    return int(seed) + 1000 * int(rank)


def batch_slice(global_batch: int, world: int, rank: int) -> range:
    """Contiguous slice of [0, global_batch) owned by `rank`; sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world or global_batch < 0:
        raise ValueError("need world > 0, 0 <= rank < world, global_batch >= 0")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats across all ranks (identity when
    torch.distributed is not initialised)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(work_per_rank: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job rate: all ranks' work over the slowest rank's time, per second."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return work_per_rank * world * steps / (max_ms / 1e3)
