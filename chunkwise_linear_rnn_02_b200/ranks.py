"""Rank bookkeeping for running the GLA operator on several GPUs, one process per GPU.

The recurrence runs along time inside one (batch, head) sequence and couples nothing across
sequences: each head keeps its own compressed matrix memory that its own gates keep, decay or
overwrite ("Gated Linear Attention for Efficient Long Sequences", "Step-by-step memory update";
"MS-GLA ...", section 2.1: the gate scales the rows of that memory), so a multi-GPU run is plain
data parallelism: every rank owns
whole sequences, computes them with the single-GPU kernels and exchanges no data.  What remains
to agree on is which rows of a batch a rank owns, which seed its synthetic batch uses, and how
the per-rank step times and token counts combine into one figure (the slowest rank sets the
step time; the tokens of all ranks add up).  `torch.distributed` carries those two scalars; it
works the same over NCCL (GPU ranks) and gloo (CPU ranks, used by the tests).
"""
from __future__ import annotations

import os
from typing import List, Sequence, Tuple


def rank_env() -> Tuple[int, int, int]:
    """(world size, global rank, local rank) from the launcher's environment (1, 0, 0 without one)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def batch_seed(base: int, rank: int) -> int:
    """Seed of a rank's synthetic batch: distinct per rank, fixed for a given base."""
    return base + rank


def shard_rows(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, stop) share of n batch rows for `rank`; shares differ by at most one row."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"bad shard request n={n} world={world} rank={rank}")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def _reduce(values: Sequence[float], device, op_name: str) -> List[float]:
    import torch
    import torch.distributed as dist

    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=getattr(dist.ReduceOp, op_name))
    return t.tolist()


def max_over_ranks(values: Sequence[float], device="cpu") -> List[float]:
    """Element-wise maximum over all ranks (every rank must call it, with the same length)."""
    return _reduce(values, device, "MAX")


def sum_over_ranks(values: Sequence[float], device="cpu") -> List[float]:
    """Element-wise sum over all ranks (every rank must call it, with the same length)."""
    return _reduce(values, device, "SUM")
