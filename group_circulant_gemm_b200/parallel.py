"""Data-parallel plumbing over torch.distributed (rows are independent).

The layer's forward and input gradient shard over the N rows with no exchange
at all; the weight gradient of a row-sharded batch is the sum over ranks of
each rank's partial dW (and dbias), one all-reduce.  These helpers hold that
host logic; the arithmetic runs in the CUDA library on each rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def row_shard(N: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced [start, stop) slice of N rows for `rank` of `world`."""
    if world < 1 or not 0 <= rank < world or N < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(N, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank scalar (timings are reported as the slowest rank)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_weight_grad(dW: torch.Tensor, dbias: torch.Tensor | None = None):
    """Sum per-rank partial weight gradients in FP32; returns tensors in dW's dtype."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return dW, dbias
    acc = dW.float()
    dist.all_reduce(acc, op=dist.ReduceOp.SUM)
    out_b = None
    if dbias is not None:
        bacc = dbias.float()
        dist.all_reduce(bacc, op=dist.ReduceOp.SUM)
        out_b = bacc.to(dbias.dtype)
    return acc.to(dW.dtype), out_b
