"""Data-parallel plumbing over torch.distributed (rows are independent).

The layer's forward and input gradient shard over the N rows with no exchange
at all; the weight gradient of a row-sharded batch is the sum over ranks of
each rank's partial dW (and dbias), one all-reduce.  Each rank writes its FP32
sums into one flat buffer (``EqLinearPlan.backward_weight_f32``), the buffer is
summed over ranks in FP32, and one cast rounds it (``cast_from_f32``), so the
ranks' contributions meet before the single rounding a one-rank run has.
These helpers hold that host logic; the arithmetic runs in the CUDA library on
each rank.
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


def allreduce_grad_buffer(buf: torch.Tensor, async_op: bool = False):
    """Sum a flat FP32 gradient buffer (dW then dbias) over ranks, in place.

    With ``async_op`` the reduction is queued behind the work already on the
    current stream and a handle is returned; ``handle.wait()`` makes the current
    stream wait for it, so independent kernels (dX) can run in between.  Returns
    None when there is nothing to reduce (one rank).
    """
    if buf.dtype != torch.float32:
        raise ValueError("the data-parallel gradient is reduced in FP32")
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return None
    return dist.all_reduce(buf, op=dist.ReduceOp.SUM, async_op=async_op)
