"""Row sharding across ranks, one process per GPU.

The rotation acts on every row independently (HARP technical summary §2.1: the
transform is applied row by row), so a batch is split into contiguous row blocks, the
plan is replicated on every rank, and the data path needs no collective.  The only
cross-rank traffic is host plumbing: a barrier around timed regions and the maximum
of the per-rank device times.
"""
from __future__ import annotations

from typing import Tuple


def weak_shard(rows_per_rank: int, rank: int) -> Tuple[int, int]:
    """(first row, row count) of `rank` when every rank gets the same number of rows
    (weak scaling: the global batch is world * rows_per_rank)."""
    if rows_per_rank < 0 or rank < 0:
        raise ValueError("negative rows or rank")
    return rank * rows_per_rank, rows_per_rank


def strong_shard(total_rows: int, world: int, rank: int) -> Tuple[int, int]:
    """(first row, row count) of `rank` when `total_rows` are split over `world` ranks
    in contiguous blocks whose sizes differ by at most one (strong scaling)."""
    if world <= 0 or not 0 <= rank < world or total_rows < 0:
        raise ValueError("bad world, rank or row count")
    base, extra = divmod(total_rows, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The maximum of `value` over all ranks (the identity without a process group).
    With NCCL, `device` is this rank's CUDA device; with gloo it is the CPU."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
