"""Data-parallel use of the head: token rows sharded over ranks, W replicated.

Rows are independent once the mean's denominator is known, so each rank runs
the fused head on its own tokens with the mean taken over the valid targets of
*every* rank; the ranks' losses then add up to the batch loss and their dW to
the batch dW, while each rank's dX is already final for its rows.  The
exchanges are one all-reduce of the count (before the call) and all-reduces of
the loss and dW (after it), through torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _device_call(X, W, y, ignore_index, mean_count):
    from .flce import forward_backward_ex
    loss, status, _, dX, dW = forward_backward_ex(X, W, y, ignore_index, mean_count=mean_count)
    return loss, status, dX, dW


def dp_forward_backward(X, W, y, ignore_index: int = -100, *, group=None, local_call=None):
    """Returns (batch loss, this rank's dX, batch dW) for this rank's shard.

    ``local_call(X, W, y, ignore_index, mean_count) -> (loss[1], status[1], dX, dW)``
    runs the head on the shard with the mean over ``mean_count`` valid targets;
    it defaults to the CUDA library.
    """
    call = local_call or _device_call
    n = (y != ignore_index).sum().to(torch.int32).reshape(1)
    dist.all_reduce(n, op=dist.ReduceOp.SUM, group=group)
    loss, status, dX, dW = call(X, W, y, ignore_index, n)
    bad = status.to(torch.int32).reshape(1).clone()
    dist.all_reduce(bad, op=dist.ReduceOp.MAX, group=group)
    if int(bad.item()) != 0:
        from .flce import FlceError
        raise FlceError(int(bad.item()), "dp_forward_backward")
    dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(dW, op=dist.ReduceOp.SUM, group=group)
    return loss, dX, dW
