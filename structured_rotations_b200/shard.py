"""Sharding across ranks, one process per GPU.

The rotation acts on every row independently (HARP technical summary §2.1: the
transform is applied row by row), so a batch is split into contiguous row blocks, the
plan is replicated on every rank, and the data path needs no collective; the only
cross-rank traffic is host plumbing (a barrier around timed regions and the maximum of
the per-rank device times).  The two-sided weight rotation of a row-sharded weight does
have an exchange: its column side needs whole columns (two_sided_row_sharded).
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


def two_sided_row_sharded(plan_u, plan_v, w_local, group=None, *, work_dtype=None, row_fn=None, col_fn=None):
    """W_out = T_U^T W T_V for a weight W whose rows are split over the ranks of `group` in
    equal contiguous blocks (rank r holds rows [r n, (r+1) n), n = n_out / world); returns
    this rank's rows of W_out.  Rows of W take T_V^T and columns T_U^T (HARP abstract: a
    rotation on each side of a weight matrix):

      1. rows, local: z = T_V^T applied to every local row (harp_apply_ex, fp32 out);
      2. one all-to-all: rank r sends rank j the j-th block of n_in / world columns of its
         rows, and receives every rank's rows of its own column block, i.e. n_out whole
         columns;
      3. columns, local: T_U^T on every column of the block (harp_apply_columns, rounded to
         W's type);
      4. one all-to-all back to the row blocks.

    The two exchanges are the only collectives; each moves (world - 1) / world of the
    rank's share.  `row_fn(src, dst)` and `col_fn(src, dst)` replace the two library calls
    (tests run the exchange on CPU ranks with a float64 reference in their place);
    `work_dtype` is the intermediate's type (float32 by default)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group) if dist.is_initialized() else 1
    n_local, n_in = w_local.shape
    if n_in % world:
        raise ValueError("the number of columns must be a multiple of the number of ranks")
    c = n_in // world
    n_out = n_local * world
    work_dtype = work_dtype or torch.float32
    z = torch.empty(n_local, n_in, dtype=work_dtype, device=w_local.device)
    if row_fn is None:
        plan_v.apply_ex(w_local, z, direction="inverse")
    else:
        row_fn(w_local, z)
    send = z.view(n_local, world, c).transpose(0, 1).contiguous()       # [world][n_local][c]
    recv = torch.empty_like(send)
    if world > 1:
        dist.all_to_all_single(recv, send, group=group)
    else:
        recv.copy_(send)
    cols = recv.view(n_out, c)                                           # rows in global order
    res = torch.empty(n_out, c, dtype=w_local.dtype, device=w_local.device)
    if col_fn is None:
        plan_u.apply_columns(cols, res, direction="inverse")
    else:
        col_fn(cols, res)
    back = torch.empty_like(res.view(world, n_local, c))
    if world > 1:
        dist.all_to_all_single(back, res.view(world, n_local, c).contiguous(), group=group)
    else:
        back.copy_(res.view(world, n_local, c))
    return back.transpose(0, 1).reshape(n_local, n_in)


def grad_theta_sharded(plan, x_local, g_local, group=None, *, grad_fn=None):
    """dL/dtheta for L = sum_r g_r . (T x_r) over the rows of every rank of `group`, each rank
    holding its own rows x_local and upstream gradients g_local (HARP technical summary §2.3:
    theta is fitted from calibration data, spread here over the ranks).  Each rank forms the
    gradient of its rows (harp_grad_theta), then one all-reduce sums them, so every rank
    ends with the same dL/dtheta.  `grad_fn(x, g)` replaces the library call (tests run the
    exchange on CPU ranks with a float64 reference in its place)."""
    import torch.distributed as dist

    d = plan.grad_theta(x_local, g_local) if grad_fn is None else grad_fn(x_local, g_local)
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(d, op=dist.ReduceOp.SUM, group=group)
    return d
