"""Plain fp64 CPU oracle for the fused linear + cross-entropy (FLCE) head.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
the benchmark's CPU-baseline leg may import this module; the product path never
does, and this module imports nothing from the product.

What it computes is the unfused definition written out in fp64.  The pages say
the fused head returns the same loss as the plain "linear layer, then
cross-entropy" pipeline, only without keeping the logit tensor:

* "Liger-Kernel: Triton kernels that replace HF training ops", section "What
  actually gets replaced": FusedLinearCrossEntropy takes the hidden states and
  the LM-head weight and returns the loss directly, a drop-in replacement with
  the same call signature.
* "Liger Kernel explained", section on the cross-entropy head: the loss and its
  gradient are computed in chunks over the vocabulary, so the full logit tensor
  is never resident; a naive head materialises it once for the forward softmax
  and once more for the gradient.
* "Complete Guide to Liger Kernel", section LigerFusedLinearCrossEntropyLoss:
  ``loss = fused_loss_fn(hidden_states, weight, labels)`` with ``weight`` of
  shape ``(vocab_size, hidden_size)``.
* The same guide, section LigerCrossEntropyLoss: cross-entropy computed from a
  given ``(batch*seq, vocab)`` logit tensor and labels (:func:`ce_reference`).
* "Liger-Kernel: Triton kernels that replace HF training ops", section
  "Installation and the one-line patch": the fused-linear post-training losses
  (ORPO, DPO, ...) take the LM-head weight, the hidden states and the targets
  and return the loss; :func:`pairwise_logistic` is the DPO-form loss on the
  per-sequence log-probabilities that the head's row losses give.

The oracle therefore *does* materialise the logits (that is the plain
definition) and follows these steps, with ``n`` the number of non-ignored rows:

1. ``valid_i = (y_i != ignore_index)``; a valid ``y_i`` outside ``[0, V)`` is an
   error.
2. ``z_ij = x_i . w_j``; ``lse_i = m_i + log(sum_j exp(z_ij - m_i))`` with
   ``m_i = max_j z_ij``; ``l_i = lse_i - z_{i, y_i}``.
3. ``loss = (sum over valid i of l_i) / n``  (token mean, the PyTorch
   ``reduction='mean'`` convention a drop-in replacement implies).
4. ``G_ij = valid_i * (exp(z_ij - lse_i) - [j == y_i]) / n``  (d loss / d z).
5. ``dX = G W``  and  ``dW = G^T X``.

Readings where the pages are silent: the mean runs over non-ignored rows; with
no valid row the loss, dX and dW are all zero (PyTorch would give NaN); there is
no bias, label smoothing, soft-cap or z-loss term.

Reductions.  A drop-in replacement of the unfused head (same call signature)
also offers PyTorch's other reductions; the oracle writes all three as one
weighted sum over valid rows, ``loss = sum_valid s_i l_i`` with
``s_i = 1/n`` ('mean'), ``1`` ('sum') or the caller's per-row upstream gradient
``g_i`` ('none', default 1), and ``G_ij = s_i (exp(z_ij - lse_i) - [j == y_i])``
for valid rows, so that dX and dW are the gradients of that loss.

Vocabulary shards.  Because the loss is computed chunk by chunk over the
vocabulary (second page above), the chunks may live on different devices: a
shard of W rows ``[v0, v0 + V_s)`` yields, per row, the log-sum-exp of its own
logits and the target logit when the target falls inside it
(:func:`shard_stats`); the log-sum-exp of the shards' values is ``lse_i`` and
the sum of their target logits is ``z_{i, y_i}`` (:func:`merge_shard_stats`).
Each shard's columns of G then give its rows of dW in full and its share of dX.

Inputs are converted exactly to fp64 (bf16 -> fp64 is exact).  A matrix product
(numpy/BLAS in fp64) serves as a step; nothing is blocked, fused or reordered
beyond what the definition states, except that the functions meant for full-size
workloads (:func:`full_loss`, :func:`full_grads` and the row-subset functions)
evaluate the per-row definition for a block of rows at a time so that the fp64
logits of a block, not of the whole batch, are in memory.
"""
from __future__ import annotations

import numpy as np

IGNORE_INDEX = -100


class TargetOutOfRange(ValueError):
    """A non-ignored target lies outside [0, V)."""


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # a torch tensor; bf16 -> fp32 -> fp64 is exact
        a = a.detach().to("cpu")
        if str(a.dtype) in ("torch.bfloat16", "torch.float16"):
            a = a.float()
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def _i64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.asarray(a, dtype=np.int64)


def valid_mask(y: np.ndarray, V: int, ignore_index: int = IGNORE_INDEX) -> np.ndarray:
    """Step 1: which rows count, and the range check on the ones that do."""
    y = _i64(y)
    valid = y != ignore_index
    bad = valid & ((y < 0) | (y >= V))
    if bad.any():
        raise TargetOutOfRange(f"target {int(y[bad][0])} outside [0, {V})")
    return valid


def log_sum_exp(Z: np.ndarray) -> np.ndarray:
    """Step 2: lse_i = m_i + log(sum_j exp(z_ij - m_i)), m_i = max_j z_ij."""
    m = Z.max(axis=1)
    return m + np.log(np.exp(Z - m[:, None]).sum(axis=1))


def row_scale(valid: np.ndarray, reduction: str, grad_row_scale=None) -> np.ndarray:
    """Weight s_i of each row's loss in the reduced loss (0 for ignored rows)."""
    n = int(valid.sum())
    if reduction == "mean":
        s = np.full(valid.shape, (1.0 / n) if n else 0.0)
    elif reduction == "sum":
        s = np.ones(valid.shape)
    elif reduction == "none":
        s = np.ones(valid.shape) if grad_row_scale is None else _f64(grad_row_scale)
    else:
        raise ValueError(f"unknown reduction {reduction!r}")
    return np.where(valid, s, 0.0)


def flce_reference(X, W, y, ignore_index: int = IGNORE_INDEX, reduction: str = "mean", grad_row_scale=None,
                   return_rows: bool = False):
    """The whole definition on full matrices: returns (loss, dX, dW, lse, n),
    plus the per-row losses when ``return_rows``.

    For shapes whose N x V fp64 logits fit in host memory.
    """
    X = _f64(X)
    W = _f64(W)
    y = _i64(y)
    N, _ = X.shape
    V = W.shape[0]
    valid = valid_mask(y, V, ignore_index)
    n = int(valid.sum())
    rows = np.arange(N)
    yv = np.where(valid, y, 0)
    s = row_scale(valid, reduction, grad_row_scale)

    Z = X @ W.T                                   # z_ij = x_i . w_j
    lse = log_sum_exp(Z)
    row_loss = np.where(valid, lse - Z[rows, yv], 0.0)
    loss = float((s * row_loss).sum())           # mean: (sum of valid l_i) / n

    G = np.exp(Z - lse[:, None])                  # softmax
    G[rows, yv] -= 1.0                            # minus the one-hot target
    G *= s[:, None]                               # s_i: token mean (or sum / upstream weights); 0 on ignored rows
    dX = G @ W
    dW = G.T @ X
    if return_rows:
        return loss, dX, dW, lse, n, row_loss
    return loss, dX, dW, lse, n


# ---------------------------------------------------------------------------
# Full-size workloads: the same per-row definition, evaluated on chosen rows.
# ---------------------------------------------------------------------------

def row_lse(X, W, rows=None, block: int = 256, W64=None) -> np.ndarray:
    """lse_i (step 2) for the given rows (all rows when ``rows`` is None).

    Rows are independent, so each block of rows is the definition applied to
    those rows; only memory is bounded by the blocking.
    """
    X = _f64(X)
    if rows is not None:
        X = X[np.asarray(rows, dtype=np.int64)]
    W64 = _f64(W) if W64 is None else W64
    out = np.empty(X.shape[0], dtype=np.float64)
    for b in range(0, X.shape[0], block):
        out[b:b + block] = log_sum_exp(X[b:b + block] @ W64.T)
    return out


def full_loss(X, W, y, ignore_index: int = IGNORE_INDEX, block: int = 256, W64=None):
    """Step 3 over all rows without the N x V matrix: returns (loss, lse, n)."""
    W64 = _f64(W) if W64 is None else W64
    X64 = _f64(X)
    y = _i64(y)
    V = W64.shape[0]
    valid = valid_mask(y, V, ignore_index)
    n = int(valid.sum())
    lse = row_lse(X64, W64, None, block, W64)
    yv = np.where(valid, y, 0)
    zy = np.einsum("ih,ih->i", X64, W64[yv])      # z_{i, y_i}
    row_loss = np.where(valid, lse - zy, 0.0)
    loss = float(row_loss.sum() / n) if n else 0.0
    return loss, lse, n


def dx_rows(X, W, y, rows, lse_rows, n: int, ignore_index: int = IGNORE_INDEX, W64=None):
    """Steps 4-5 for the chosen token rows: dX_i = sum_j G_ij w_j."""
    W64 = _f64(W) if W64 is None else W64
    rows = np.asarray(rows, dtype=np.int64)
    Xr = _f64(X)[rows]
    yr = _i64(y)[rows]
    V = W64.shape[0]
    valid = valid_mask(yr, V, ignore_index)
    Z = Xr @ W64.T
    G = np.exp(Z - np.asarray(lse_rows, dtype=np.float64)[:, None])
    G[np.arange(len(rows)), np.where(valid, yr, 0)] -= 1.0
    G *= valid[:, None]
    G *= (1.0 / n) if n else 0.0
    return G @ W64


def dw_rows(X, W, y, vocab_rows, lse, n: int, ignore_index: int = IGNORE_INDEX, W64=None, X64=None):
    """Steps 4-5 for the chosen vocab entries: dW_j = sum_i G_ij x_i.

    Needs lse_i for every token row (from :func:`full_loss`).
    """
    W64 = _f64(W) if W64 is None else W64
    X64 = _f64(X) if X64 is None else X64
    y = _i64(y)
    J = np.asarray(vocab_rows, dtype=np.int64)
    V = W64.shape[0]
    valid = valid_mask(y, V, ignore_index)
    Z = X64 @ W64[J].T                            # z_ij for all i, chosen j
    G = np.exp(Z - np.asarray(lse, dtype=np.float64)[:, None])
    G -= (y[:, None] == J[None, :])               # one-hot at the target
    G *= valid[:, None]
    G *= (1.0 / n) if n else 0.0
    return G.T @ X64


def full_grads(X, W, y, ignore_index: int = IGNORE_INDEX, block: int = 1024, W64=None, X64=None):
    """Steps 1-5 over every row and every vocabulary entry, with the 'mean'
    reduction: returns (loss, dX, dW, lse, n) like :func:`flce_reference`.

    The rows are taken a block at a time.  For the rows b of a block the logits
    Z_b = X_b W^T, their lse, their row losses and G_b follow the definition
    exactly as for the whole matrix; dX_b = G_b W is final for those rows, and
    dW = sum over blocks of G_b^T X_b (the same sum over rows as G^T X, grouped
    by block).  Only the fp64 logits of one block are in memory at a time.
    """
    W64 = _f64(W) if W64 is None else W64
    X64 = _f64(X) if X64 is None else X64
    y = _i64(y)
    N = X64.shape[0]
    V = W64.shape[0]
    valid = valid_mask(y, V, ignore_index)
    n = int(valid.sum())
    inv_n = (1.0 / n) if n else 0.0
    dX = np.empty_like(X64)
    dW = np.zeros_like(W64)
    lse = np.empty(N, dtype=np.float64)
    loss_sum = 0.0
    for b0 in range(0, N, block):
        b1 = min(N, b0 + block)
        rows = np.arange(b1 - b0)
        vb = valid[b0:b1]
        yb = np.where(vb, y[b0:b1], 0)
        Z = X64[b0:b1] @ W64.T                     # z_ij for the block's rows
        lse_b = log_sum_exp(Z)
        loss_sum += float(np.where(vb, lse_b - Z[rows, yb], 0.0).sum())
        Z -= lse_b[:, None]                        # G_b, in place of the block's logits:
        np.exp(Z, out=Z)                           #   softmax
        Z[rows, yb] -= 1.0                         #   minus the one-hot target
        Z *= (vb * inv_n)[:, None]                 #   1/n on valid rows, 0 on ignored rows
        dX[b0:b1] = Z @ W64
        dW += Z.T @ X64[b0:b1]
        lse[b0:b1] = lse_b
    loss = float(loss_sum / n) if n else 0.0
    return loss, dX, dW, lse, n


# ---------------------------------------------------------------------------
# Cross-entropy on given logits (no linear layer).
# ---------------------------------------------------------------------------

def ce_reference(Z, y, ignore_index: int = IGNORE_INDEX, reduction: str = "mean", grad_row_scale=None):
    """Steps 1-4 on a given logit matrix Z[N,V]: returns (loss, dZ, lse, n, row_loss).

    dZ = G is the gradient of the reduced loss with respect to the logits.
    """
    Z = _f64(Z)
    y = _i64(y)
    N, V = Z.shape
    valid = valid_mask(y, V, ignore_index)
    n = int(valid.sum())
    rows = np.arange(N)
    yv = np.where(valid, y, 0)
    s = row_scale(valid, reduction, grad_row_scale)
    lse = log_sum_exp(Z)
    row_loss = np.where(valid, lse - Z[rows, yv], 0.0)
    loss = float((s * row_loss).sum())
    G = np.exp(Z - lse[:, None])
    G[rows, yv] -= 1.0
    G *= s[:, None]
    return loss, G, lse, n, row_loss


def shard_stats(X, W_shard, y, v0: int, ignore_index: int = IGNORE_INDEX):
    """Statistics of one vocabulary shard, W rows ``v0 .. v0 + V_s - 1`` given as
    ``W_shard``: returns ``(lse_s, zy_s)`` with ``lse_s[i]`` the log-sum-exp of
    row i's logits over the shard and ``zy_s[i]`` its target logit when
    ``v0 <= y_i < v0 + V_s`` (0 otherwise, and for ignored rows).  The global
    range of the targets is the caller's to check."""
    X = _f64(X)
    Ws = _f64(W_shard)
    y = _i64(y)
    Z = X @ Ws.T                                   # this shard's logits
    lse_s = log_sum_exp(Z)
    local = y - v0
    inside = (y != ignore_index) & (local >= 0) & (local < Ws.shape[0])
    zy_s = np.where(inside, Z[np.arange(len(y)), np.where(inside, local, 0)], 0.0)
    return lse_s, zy_s


def merge_shard_stats(all_lse, all_zy):
    """Merges the shards' statistics, arrays ``[shards][N]``: ``lse_i`` is the
    log-sum-exp over shards of their log-sum-exps (exact: the exponential sums
    add), and ``z_{i, y_i}`` the sum of their target logits (one shard holds
    the target).  Returns ``(lse, zy)``."""
    L = _f64(all_lse)
    return log_sum_exp(L.T), _f64(all_zy).sum(axis=0)


# ---------------------------------------------------------------------------
# Pairwise logistic (DPO-form) preference loss on the head's row losses.
# ---------------------------------------------------------------------------

def pairwise_logistic(row_loss, y, seq_start, chosen, rejected, beta: float, ref_logp=None,
                      ignore_index: int = IGNORE_INDEX):
    """Sequence s holds the token rows ``seq_start[s] .. seq_start[s+1]-1``;
    ``logp_s = -(sum of their row losses)`` (a row loss is -log p(y_i | x_i),
    0 on ignored rows).  Pair k compares sequences ``chosen[k]`` and
    ``rejected[k]``: ``m_k = beta ((logp_c - ref_c) - (logp_r - ref_r))`` and
    ``L = -(1/P) sum_k log sigmoid(m_k)``.  Returns
    ``(L, logp, dL/dlogp, row weights)`` where the weight of a valid row i of
    sequence s is ``-dL/dlogp_s`` (the upstream gradient of its row loss) and
    every other row's is 0."""
    rl = _f64(row_loss)
    y = _i64(y)
    st = _i64(seq_start)
    c = _i64(chosen)
    r = _i64(rejected)
    S = len(st) - 1
    logp = np.array([-rl[st[s]:st[s + 1]].sum() for s in range(S)])
    d = logp if ref_logp is None else logp - _f64(ref_logp)
    m = beta * (d[c] - d[r])
    P = len(c)
    loss = float(np.logaddexp(0.0, -m).sum() / P)       # -log sigmoid(m) = log(1 + e^-m)
    gm = -1.0 / (1.0 + np.exp(m)) / P                   # dL/dm_k = -sigmoid(-m_k) / P
    grad = np.zeros(S)
    for k in range(P):
        grad[c[k]] += beta * gm[k]
        grad[r[k]] -= beta * gm[k]
    w = np.zeros(len(rl))
    for s in range(S):
        w[st[s]:st[s + 1]] = -grad[s]
    w[y == ignore_index] = 0.0
    return loss, logp, grad, w
