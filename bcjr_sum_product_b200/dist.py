"""Data-parallel helpers: sequences are independent, so a multi-GPU run gives
each rank a contiguous slice of the sequences; the only exchange is the sum of
the codebook gradient over ranks (one all-reduce of 2^L * V floats per VJP).

The local computation is a parameter so that the host logic can be exercised
with CPU ranks (gloo) and any local implementation.
"""
from __future__ import annotations

from typing import Callable, Tuple

import torch
import torch.distributed as dist


def shard_rows(n_seq: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) slice of rank ``rank``; sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n_seq, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def vjp_data_parallel(local_vjp: Callable, w_local, codebook, grad_soft_local, group=None):
    """Runs ``local_vjp(w_local, codebook, grad_soft_local) -> (grad_w_local, grad_codebook_local)``
    and sums the codebook gradient over the ranks of ``group`` in place.
    Returns (grad_w_local, grad_codebook_total)."""
    gw, gc = local_vjp(w_local, codebook, grad_soft_local)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(gc, op=dist.ReduceOp.SUM, group=group)
    return gw, gc


def max_over_ranks(value: float, device=None, group=None) -> float:
    """Maximum of a per-rank timing over the ranks (the multi-GPU step time)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t[0])
