"""Multi-device use of the head: data-parallel over tokens, or vocabulary-parallel.

Data-parallel (:func:`dp_forward_backward`): token rows sharded over ranks, W
replicated.

Rows are independent once the mean's denominator is known, so each rank runs
the fused head on its own tokens with the mean taken over the valid targets of
*every* rank; the ranks' losses then add up to the batch loss and their dW to
the batch dW, while each rank's dX is already final for its rows.  The
exchanges are one all-reduce of the count (before the call) and all-reduces of
the loss and dW (after it), through torch.distributed (NCCL on GPUs).  With
``overlap_sections`` the gradient pass runs in sections of whole vocabulary
chunks and each section's finished dW rows are all-reduced on a second stream
while the later sections compute (:func:`dp_forward_backward_overlapped`).

Vocabulary-parallel (:func:`vp_forward_backward`): W rows sharded over ranks in
contiguous ranges, X and y replicated.  The loss is computed chunk by chunk
over the vocabulary, so each rank reduces its own chunk to per-row statistics
(log-sum-exp, target logit); one all-gather of those two N-vectors gives every
rank the global log-sum-exp, after which its dW rows are complete and its dX is
a share that one all-reduce sums.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _device_call(X, W, y, ignore_index, mean_count):
    from .flce import forward_backward_ex
    loss, status, _, dX, dW = forward_backward_ex(X, W, y, ignore_index, mean_count=mean_count)
    return loss, status, dX, dW


def _device_count(y, ignore_index):
    from .flce import count_valid
    return count_valid(y, ignore_index)


def dp_forward_backward(X, W, y, ignore_index: int = -100, *, group=None, local_call=None, count_call=None):
    """Returns (batch loss, this rank's dX, batch dW) for this rank's shard.

    ``count_call(y, ignore_index) -> int32[1]`` counts the shard's valid
    targets and ``local_call(X, W, y, ignore_index, mean_count) -> (loss[1],
    status[1], dX, dW)`` runs the head on the shard with the mean over
    ``mean_count`` valid targets; both default to the CUDA library.
    """
    call = local_call or _device_call
    count = count_call or _device_count
    n = count(y, ignore_index)
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


def dp_forward_backward_overlapped(X, W, y, ignore_index: int = -100, *, sections: int = 4, group=None,
                                  workspace=None, comm_stream=None):
    """:func:`dp_forward_backward` with the dW all-reduce overlapped with the
    gradient pass (CUDA library and NCCL only): the call's gradient pass runs
    in ``sections`` launches; after each one, ``comm_stream`` waits for it and
    all-reduces the dW rows it finished, while the next section computes.
    Returns (batch loss, this rank's dX, batch dW) like the unsplit version."""
    from .flce import FlceError, count_valid, forward_backward_sections
    n = count_valid(y, ignore_index)
    dist.all_reduce(n, op=dist.ReduceOp.SUM, group=group)
    loss, status, dX, dW, events, rows = forward_backward_sections(X, W, y, ignore_index, sections=sections,
                                                                   mean_count=n, workspace=workspace)
    main = torch.cuda.current_stream(X.device)
    comm = comm_stream or torch.cuda.Stream(device=X.device)
    with torch.cuda.stream(comm):
        for k, ev in enumerate(events):
            comm.wait_event(ev)
            if rows[k + 1] > rows[k]:
                dist.all_reduce(dW[rows[k]:rows[k + 1]], op=dist.ReduceOp.SUM, group=group)
    main.wait_stream(comm)
    bad = status.clone()
    dist.all_reduce(bad, op=dist.ReduceOp.MAX, group=group)
    if int(bad.item()) != 0:
        raise FlceError(int(bad.item()), "dp_forward_backward_overlapped")
    dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=group)
    return loss, dX, dW


def _vp_stats_call(X, W_shard, y, v0, V, ignore_index):
    from .flce import vp_shard_stats
    return vp_shard_stats(X, W_shard, y, v0, V, ignore_index)


def _vp_backward_call(X, W_shard, y, v0, V, all_lse, all_zy, ignore_index):
    from .flce import vp_backward
    return vp_backward(X, W_shard, y, v0, V, all_lse, all_zy, ignore_index)


def vocab_shard_range(V: int, world: int, rank: int):
    """The contiguous W rows ``[v0, v1)`` rank ``rank`` of ``world`` holds: the
    vocabulary split as evenly as possible, the first ``V % world`` shards one
    row longer."""
    base, extra = divmod(V, world)
    v0 = rank * base + min(rank, extra)
    return v0, v0 + base + (1 if rank < extra else 0)


def vp_forward_backward(X, W_shard, y, v0: int, V: int, ignore_index: int = -100, *, group=None,
                        stats_call=None, backward_call=None):
    """Returns (loss, dX, dW_shard) on every rank of ``group`` for a vocabulary
    split into contiguous shards; this rank holds W rows ``[v0, v0 + V_s)``.

    ``stats_call(X, W_shard, y, v0, V, ignore_index) -> (lse[N], zy[N], status[1])``
    and ``backward_call(X, W_shard, y, v0, V, all_lse, all_zy, ignore_index) ->
    (loss[1], status[1], dX_part, dW_shard)`` default to the CUDA library.
    """
    stats = stats_call or _vp_stats_call
    back = backward_call or _vp_backward_call
    world = dist.get_world_size(group)
    lse, zy, st1 = stats(X, W_shard, y, v0, V, ignore_index)
    both = torch.stack([lse, zy])                                   # [2, N]
    gathered = [torch.empty_like(both) for _ in range(world)]
    dist.all_gather(gathered, both, group=group)
    allst = torch.stack(gathered)                                   # [world, 2, N]
    all_lse = allst[:, 0].contiguous()
    all_zy = allst[:, 1].contiguous()
    loss, st2, dX, dW = back(X, W_shard, y, v0, V, all_lse, all_zy, ignore_index)
    bad = torch.maximum(st1.to(torch.int32).reshape(1), st2.to(torch.int32).reshape(1)).clone()
    dist.all_reduce(bad, op=dist.ReduceOp.MAX, group=group)
    if int(bad.item()) != 0:
        from .flce import FlceError
        raise FlceError(int(bad.item()), "vp_forward_backward")
    dist.all_reduce(dX, op=dist.ReduceOp.SUM, group=group)
    return loss, dX, dW
