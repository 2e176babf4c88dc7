"""Fused-linear preference loss on top of the head.

The post-training losses of the library the pages describe ("Liger-Kernel:
Triton kernels that replace Hugging Face training ops", section "Installation
and the one-line patch": ORPO called with the LM-head weight, the hidden states
and the targets, returning the loss directly; DPO, CPO, SimPO and others
listed) all need the same two things from the LM head, without the N x V
logits: the log-probability of each target token, and the gradient of a loss
built from their per-sequence sums.  Both come from the fused head:

1. one forward-only call with per-row losses gives log p(y_i | x_i) = -l_i;
2. each sequence s sums its rows: logp_s = sum_{i in s} -l_i;
3. the preference loss over (chosen, rejected) pairs, here the logistic
   (DPO-form) loss  L = -(1/P) sum_k log sigmoid(beta * (d_c - d_r)),  with
   d = logp - ref_logp (reference log-probabilities optional, 0 by default),
   gives dL/dlogp_s on the S sequences;
4. one full call with reduction 'none' and per-row upstream weights
   w_i = -dL/dlogp_{seq(i)} gives dX and dW, because d logp_s / d z_i =
   -(softmax_i - onehot_i) for the rows of s.

Steps 2-3 touch only S numbers and N row losses; the two head calls do all the
work on X and W.
"""
from __future__ import annotations

import torch


def _head_rows(X, W, y, ignore_index):
    from .flce import forward_backward_ex
    _, status, row_loss, _, _ = forward_backward_ex(X, W, y, ignore_index, reduction="none", row_loss=True,
                                                    grads=False)
    return row_loss, status


def _head_grads(X, W, y, ignore_index, weights):
    from .flce import forward_backward_ex
    _, status, _, dX, dW = forward_backward_ex(X, W, y, ignore_index, reduction="none", grad_row_scale=weights)
    return dX, dW, status


def sequence_logps(row_loss, seq, num_seqs: int):
    """logp_s = -sum of the row losses of sequence s (ignored rows have 0)."""
    out = torch.zeros(num_seqs, dtype=torch.float64, device=row_loss.device)
    return out.index_add_(0, seq, -row_loss.to(torch.float64))


def pairwise_logistic(logp, chosen, rejected, beta: float, ref_logp=None):
    """L = -(1/P) sum_k log sigmoid(beta * ((logp_c - ref_c) - (logp_r - ref_r)))
    over the P pairs (chosen[k], rejected[k]); returns (L, dL/dlogp) in fp64."""
    d = logp if ref_logp is None else logp - ref_logp.to(logp.dtype)
    margin = beta * (d[chosen] - d[rejected])
    P = chosen.numel()
    loss = -torch.nn.functional.logsigmoid(margin).sum() / P
    # d(-log sigmoid(m))/dm = -sigmoid(-m)
    gm = -torch.sigmoid(-margin) / P
    grad = torch.zeros_like(logp)
    grad.index_add_(0, chosen, beta * gm)
    grad.index_add_(0, rejected, -beta * gm)
    return loss, grad


def preference_forward_backward(X, W, y, seq, chosen, rejected, beta: float = 0.1, ref_logp=None,
                                ignore_index: int = -100, *, head_rows=None, head_grads=None):
    """Pairwise logistic preference loss of sequences packed as token rows.

    X [N, H], W [V, H], y [N] (prompt and padding rows = ignore_index); seq [N]
    int64: the sequence of each row; chosen / rejected [P] int64: sequence ids
    of each pair; ref_logp [S] or None.  Returns (loss, dX, dW, logp).

    ``head_rows(X, W, y, ignore_index) -> (row_loss[N], status)`` and
    ``head_grads(X, W, y, ignore_index, weights[N]) -> (dX, dW, status)``
    default to the CUDA library.
    """
    rows = head_rows or _head_rows
    grads = head_grads or _head_grads
    num_seqs = int(seq.max().item()) + 1 if seq.numel() else 0
    row_loss, st1 = rows(X, W, y, ignore_index)
    logp = sequence_logps(row_loss, seq, num_seqs)
    loss, g = pairwise_logistic(logp, chosen, rejected, beta, ref_logp)
    # d logp_s / d l_i = -1 for the rows of s: upstream weight of row i is -g_s
    weights = (-g[seq]).to(torch.float32)
    weights = torch.where(y != ignore_index, weights, torch.zeros_like(weights)).contiguous()
    dX, dW, st2 = grads(X, W, y, ignore_index, weights)
    bad = int(torch.maximum(st1.to(torch.int32).reshape(1), st2.to(torch.int32).reshape(1)).item())
    if bad:
        from .flce import FlceError
        raise FlceError(bad, "preference_forward_backward")
    return loss, dX, dW, logp
