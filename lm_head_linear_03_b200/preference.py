"""Fused-linear preference loss on top of the head.

The post-training losses of the library the pages describe ("Liger-Kernel:
Triton kernels that replace Hugging Face training ops", section "Installation
and the one-line patch": ORPO called with the LM-head weight, the hidden states
and the targets, returning the loss directly; DPO, CPO, SimPO and others
listed) all need the same two things from the LM head, without the N x V
logits: the log-probability of each target token, and the gradient of a loss
built from their per-sequence sums.  Every step runs in the CUDA library:

1. one forward-only head call with per-row losses gives log p(y_i | x_i) = -l_i;
2. flce_pairwise_logistic sums each sequence's rows, logp_s = sum_{i in s} -l_i,
   forms the logistic (DPO-form) loss over (chosen, rejected) pairs,
   L = -(1/P) sum_k log sigmoid(beta * (d_c - d_r)) with d = logp - ref_logp
   (reference log-probabilities optional, 0 by default), and turns dL/dlogp_s
   into the upstream weight w_i = -dL/dlogp_{seq(i)} of each valid row;
3. one full head call with reduction 'none' and those weights gives dX and
   dW, because d logp_s / d z_i = -(softmax_i - onehot_i) for the rows of s.

This module only passes device tensors between the three calls.
"""
from __future__ import annotations

import torch


def _head_rows(X, W, y, ignore_index):
    from .flce import forward_backward_ex
    _, status, row_loss, _, _ = forward_backward_ex(X, W, y, ignore_index, reduction="none", row_loss=True,
                                                    grads=False)
    return row_loss, status


def _pair_loss(row_loss, y, seq_start, chosen, rejected, beta, ref_logp, ignore_index):
    from .flce import pairwise_logistic
    return pairwise_logistic(row_loss, y, seq_start, chosen, rejected, beta, ref_logp, ignore_index)


def _head_grads(X, W, y, ignore_index, weights):
    from .flce import forward_backward_ex
    _, status, _, dX, dW = forward_backward_ex(X, W, y, ignore_index, reduction="none", grad_row_scale=weights)
    return dX, dW, status


def preference_forward_backward(X, W, y, seq_start, chosen, rejected, beta: float = 0.1, ref_logp=None,
                                ignore_index: int = -100, *, head_rows=None, pair_loss=None, head_grads=None):
    """Pairwise logistic preference loss of sequences packed as token rows.

    X [N, H], W [V, H], y [N] int32 (prompt and padding rows = ignore_index);
    seq_start [S+1] int32: sequence s holds rows seq_start[s] .. seq_start[s+1]-1;
    chosen / rejected [P] int32: sequence ids of each pair; ref_logp [S] fp64
    or None.  Returns (loss fp64[1], dX, dW, logp fp64[S]).

    ``head_rows(X, W, y, ignore_index) -> (row_loss[N], status)``,
    ``pair_loss(row_loss, y, seq_start, chosen, rejected, beta, ref_logp,
    ignore_index) -> (loss, logp, grad_logp, row_weight, status)`` and
    ``head_grads(X, W, y, ignore_index, weights[N]) -> (dX, dW, status)``
    default to the CUDA library.
    """
    rows = head_rows or _head_rows
    pair = pair_loss or _pair_loss
    grads = head_grads or _head_grads
    row_loss, st1 = rows(X, W, y, ignore_index)
    loss, logp, _, weights, st2 = pair(row_loss, y, seq_start, chosen, rejected, beta, ref_logp, ignore_index)
    dX, dW, st3 = grads(X, W, y, ignore_index, weights)
    statuses = [int(s.reshape(-1)[0].item()) for s in (st1, st2, st3)]
    bad = next((s for s in statuses if s), 0)
    if bad:
        from .flce import FlceError
        raise FlceError(bad, "preference_forward_backward")
    return loss, dX, dW, logp
