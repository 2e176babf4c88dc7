"""Checks that pin the fp64 oracle to facts outside itself.

Each ``pin_*`` takes the oracle module and raises ``AssertionError`` when the
module disagrees with a closed form, a textbook special case, a library routine
used as a brute force (torch fp64 cross-entropy plus autograd), central finite
differences or an invariant of the method.  ``test_oracle.py`` runs them on the
oracle; ``test_oracle_mutants.py`` runs them on copies of the oracle with one
planted mistake each and requires that some pin fails.
"""
from __future__ import annotations

import math

import numpy as np
import torch

IGN = -100


def _rng(seed):
    return np.random.default_rng(seed)


def _case(seed, N, H, V, n_ign=1, scale_x=1.0, scale_w=0.3):
    r = _rng(seed)
    X = r.standard_normal((N, H)) * scale_x
    W = r.standard_normal((V, H)) * scale_w
    y = r.integers(0, V, size=N)
    if n_ign:
        y[r.permutation(N)[:n_ign]] = IGN
    return X, W, y


def _close(a, b, rtol, atol=0.0, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    lim = atol + rtol * (np.max(np.abs(b)) if b.size else 0.0)
    assert err <= lim, f"{what}: max err {err:.3e} > {lim:.3e}"


def pin_zero_weight(orc):
    """W = 0: every logit is 0, softmax is uniform 1/V.

    loss = ln V exactly; dX = 0; dW_j = (1/n) sum_valid (1/V - [y_i = j]) x_i.
    """
    N, H, V = 7, 5, 11
    X, _, y = _case(1, N, H, V, n_ign=2)
    W = np.zeros((V, H))
    loss, dX, dW, _, n = orc.flce_reference(X, W, y)
    assert n == N - 2
    assert abs(loss - math.log(V)) <= 1e-15 * math.log(V), loss
    assert np.all(dX == 0.0)
    want = np.zeros((V, H))
    for i in range(N):
        if y[i] == IGN:
            continue
        for j in range(V):
            want[j] += ((1.0 / V) - (1.0 if y[i] == j else 0.0)) * X[i] / n
    _close(dW, want, 1e-13, what="dW at W=0")


def pin_zero_input(orc):
    """X = 0: loss = ln V, dW = 0, dX_i = valid_i (mean_j w_j - w_{y_i}) / n."""
    N, H, V = 6, 4, 9
    _, W, y = _case(2, N, H, V, n_ign=1)
    X = np.zeros((N, H))
    loss, dX, dW, _, n = orc.flce_reference(X, W, y)
    assert abs(loss - math.log(V)) <= 1e-15 * math.log(V)
    assert np.all(dW == 0.0)
    wbar = W.mean(axis=0)
    for i in range(N):
        want = np.zeros(H) if y[i] == IGN else (wbar - W[y[i]]) / n
        _close(dX[i], want, 1e-13, atol=1e-16, what=f"dX row {i} at X=0")


def pin_two_class(orc):
    """V = 2 is logistic regression: l_i = softplus(z_other - z_target),
    dX_i = sigmoid(z_other - z_target) (w_other - w_target) / n."""
    N, H = 9, 6
    X, W, y = _case(3, N, H, 2, n_ign=2, scale_w=0.8)
    loss, dX, dW, _, n = orc.flce_reference(X, W, y)
    tot = 0.0
    for i in range(N):
        if y[i] == IGN:
            assert np.all(dX[i] == 0.0)
            continue
        t, o = int(y[i]), 1 - int(y[i])
        d = float(X[i] @ W[o] - X[i] @ W[t])
        tot += max(d, 0.0) + math.log1p(math.exp(-abs(d)))
        sig = 1.0 / (1.0 + math.exp(-d))
        _close(dX[i], sig * (W[o] - W[t]) / n, 1e-12, atol=1e-15, what=f"dX row {i}, V=2")
    assert abs(loss - tot / n) <= 1e-13 * abs(tot / n), (loss, tot / n)


def pin_large_logits(orc):
    """Logits of magnitude ~1e3 overflow a naive exp; the max-shifted lse must
    stay finite and equal softplus(d) = d + log1p(exp(-d)) for V = 2."""
    X = np.array([[30.0, -20.0], [-25.0, 40.0]])
    W = np.array([[20.0, 10.0], [-15.0, 12.0]])
    y = np.array([0, 0])
    loss, dX, dW, lse, n = orc.flce_reference(X, W, y)
    tot = 0.0
    for i in range(2):
        d = float(X[i] @ W[1] - X[i] @ W[0])
        tot += max(d, 0.0) + math.log1p(math.exp(-abs(d)))
    assert np.isfinite(loss) and np.all(np.isfinite(dX)) and np.all(np.isfinite(dW))
    assert abs(loss - tot / 2) <= 1e-13 * abs(tot / 2), (loss, tot / 2)


def pin_torch_autograd(orc):
    """Brute force through another library: torch fp64 logits, torch's own
    cross_entropy(ignore_index=-100, mean) and autograd for both gradients."""
    for seed, (N, H, V, ig) in enumerate([(5, 3, 7, 1), (16, 12, 33, 4), (3, 8, 2, 0), (40, 24, 130, 7)]):
        X, W, y = _case(10 + seed, N, H, V, n_ign=ig)
        loss, dX, dW, _, _ = orc.flce_reference(X, W, y)
        tX = torch.tensor(X, dtype=torch.float64, requires_grad=True)
        tW = torch.tensor(W, dtype=torch.float64, requires_grad=True)
        ty = torch.tensor(y, dtype=torch.int64)
        tl = torch.nn.functional.cross_entropy(tX @ tW.T, ty, ignore_index=IGN, reduction="mean")
        tl.backward()
        assert abs(loss - tl.item()) <= 1e-12 * abs(tl.item()), (loss, tl.item())
        _close(dX, tX.grad.numpy(), 1e-11, what="dX vs autograd")
        _close(dW, tW.grad.numpy(), 1e-11, what="dW vs autograd")


def pin_finite_difference(orc):
    """Central differences of the loss against every entry of X and W."""
    N, H, V = 4, 8, 16
    X, W, y = _case(20, N, H, V, n_ign=1)
    _, dX, dW, _, _ = orc.flce_reference(X, W, y)
    h = 1e-5

    def L(Xa, Wa):
        return orc.flce_reference(Xa, Wa, y)[0]

    for (A, dA, is_x) in ((X, dX, True), (W, dW, False)):
        fd = np.zeros_like(A)
        for idx in np.ndindex(A.shape):
            Ap, Am = A.copy(), A.copy()
            Ap[idx] += h
            Am[idx] -= h
            lp = L(Ap, W) if is_x else L(X, Ap)
            lm = L(Am, W) if is_x else L(X, Am)
            fd[idx] = (lp - lm) / (2 * h)
        _close(dA, fd, 1e-6, atol=1e-9, what="finite differences")


def pin_rows_of_g_sum_to_zero(orc):
    """sum_j (softmax - onehot)_ij = 0 for every row, hence sum_j dW_j = 0."""
    X, W, y = _case(30, 12, 10, 50, n_ign=3)
    _, dX, dW, _, _ = orc.flce_reference(X, W, y)
    s = dW.sum(axis=0)
    assert np.max(np.abs(s)) <= 1e-13 * np.max(np.abs(dW)) * 50, s


def pin_shift_invariance(orc):
    """w_j -> w_j + c for every j adds x_i.c to a whole row of logits, which
    leaves softmax, loss and dX unchanged."""
    X, W, y = _case(40, 10, 6, 20, n_ign=2)
    c = _rng(41).standard_normal(6)
    l0, dX0, _, _, _ = orc.flce_reference(X, W, y)
    l1, dX1, _, _, _ = orc.flce_reference(X, W + c[None, :], y)
    assert abs(l0 - l1) <= 1e-12 * abs(l0)
    _close(dX1, dX0, 1e-11, atol=1e-15, what="dX under shift")


def pin_ignored_rows(orc):
    """Ignored rows give exactly zero dX, and changing their hidden state moves
    neither the loss nor dW."""
    X, W, y = _case(50, 10, 6, 20, n_ign=4)
    l0, dX0, dW0, _, _ = orc.flce_reference(X, W, y)
    ign = y == IGN
    assert np.all(dX0[ign] == 0.0)
    X2 = X.copy()
    X2[ign] += 5.0
    l1, _, dW1, _, _ = orc.flce_reference(X2, W, y)
    assert abs(l0 - l1) <= 1e-15 * abs(l0)
    _close(dW1, dW0, 1e-14, what="dW after moving ignored rows")


def pin_no_valid_rows(orc):
    """Reading for n_valid = 0: loss 0 and zero gradients."""
    X, W, _ = _case(60, 5, 4, 9, n_ign=0)
    y = np.full(5, IGN)
    loss, dX, dW, _, n = orc.flce_reference(X, W, y)
    assert n == 0 and loss == 0.0 and np.all(dX == 0) and np.all(dW == 0)


def pin_target_range(orc):
    X, W, _ = _case(61, 3, 4, 9, n_ign=0)
    for bad in (-1, 9, 1000):
        try:
            orc.flce_reference(X, W, np.array([0, bad, 2]))
        except orc.TargetOutOfRange:
            continue
        except Exception as e:  # crashed instead of reporting the bad target
            raise AssertionError(f"target {bad}: {type(e).__name__} instead of TargetOutOfRange")
        raise AssertionError(f"target {bad} accepted")


def pin_permutations(orc):
    """Relabelling the vocabulary permutes dW's rows; reordering tokens
    permutes dX's rows; neither changes the loss."""
    X, W, y = _case(70, 11, 7, 23, n_ign=2)
    l0, dX0, dW0, _, _ = orc.flce_reference(X, W, y)
    p = _rng(71).permutation(23)        # new vocab index k holds old entry p[k]
    inv = np.argsort(p)
    y2 = np.where(y == IGN, IGN, inv[np.where(y == IGN, 0, y)])
    l1, dX1, dW1, _, _ = orc.flce_reference(X, W[p], y2)
    assert abs(l0 - l1) <= 1e-13 * abs(l0)
    _close(dX1, dX0, 1e-12, atol=1e-16, what="dX under vocab relabel")
    _close(dW1, dW0[p], 1e-12, atol=1e-16, what="dW under vocab relabel")
    q = _rng(72).permutation(11)
    l2, dX2, dW2, _, _ = orc.flce_reference(X[q], W, y[q])
    assert abs(l0 - l2) <= 1e-13 * abs(l0)
    _close(dX2, dX0[q], 1e-12, atol=1e-16, what="dX under token reorder")
    _close(dW2, dW0, 1e-12, atol=1e-16, what="dW under token reorder")


def pin_equal_logits(orc):
    """All w_j equal: every row is uniform, lse_i = z_i + ln V."""
    X, _, y = _case(80, 6, 5, 13, n_ign=1)
    w = _rng(81).standard_normal(5)
    W = np.tile(w, (13, 1))
    _, _, _, lse, _ = orc.flce_reference(X, W, y)
    _close(lse, X @ w + math.log(13), 1e-14, what="lse with equal rows")


def pin_row_functions(orc):
    """The row-subset functions used at full size give what the whole-matrix
    definition gives on a case where both run."""
    X, W, y = _case(90, 300, 16, 700, n_ign=30)
    loss, dX, dW, lse, n = orc.flce_reference(X, W, y)
    l2, lse2, n2 = orc.full_loss(X, W, y, block=64)
    assert n2 == n and abs(l2 - loss) <= 1e-13 * abs(loss)
    _close(lse2, lse, 1e-14, what="row lse")
    rows = np.array([0, 5, 77, 299])
    _close(orc.dx_rows(X, W, y, rows, lse[rows], n), dX[rows], 1e-12, atol=1e-18, what="dx_rows")
    J = np.array([0, 1, 350, 699])
    _close(orc.dw_rows(X, W, y, J, lse, n), dW[J], 1e-12, atol=1e-18, what="dw_rows")
    _close(orc.row_lse(X, W, rows), lse[rows], 1e-14, what="row_lse subset")


def pin_full_grads(orc):
    """The blocked whole-tensor gradients used at full size equal the whole-matrix
    definition, on a case whose last block is ragged, one of whose blocks holds
    only ignored rows and whose targets include the first and last entries."""
    X, W, y = _case(95, 300, 24, 530, n_ign=20)
    y[64:128] = IGN          # block 1 (of 64-row blocks) is all ignored
    y[3], y[200] = 0, 529
    loss, dX, dW, lse, n = orc.flce_reference(X, W, y)
    l2, dX2, dW2, lse2, n2 = orc.full_grads(X, W, y, block=64)
    assert n2 == n and abs(l2 - loss) <= 1e-13 * abs(loss), (l2, loss)
    _close(lse2, lse, 1e-14, what="blocked lse")
    _close(dX2, dX, 1e-12, atol=1e-18, what="blocked dX")
    _close(dW2, dW, 1e-12, atol=1e-18, what="blocked dW")
    assert np.all(dX2[y == IGN] == 0.0)
    # one block covering every row, and no valid row at all
    l3, dX3, dW3, _, _ = orc.full_grads(X, W, y, block=1000)
    assert abs(l3 - loss) <= 1e-13 * abs(loss)
    _close(dW3, dW, 1e-12, atol=1e-18, what="single-block dW")
    l4, dX4, dW4, _, n4 = orc.full_grads(X, W, np.full(300, IGN), block=64)
    assert n4 == 0 and l4 == 0.0 and not dX4.any() and not dW4.any()


def _bf16_value(bits: int) -> float:
    """The number a bf16 bit pattern encodes (sign, 8-bit exponent, 7-bit
    fraction, bias 127), decoded by hand."""
    bits = int(bits)
    sign = -1.0 if bits & 0x8000 else 1.0
    e = (bits >> 7) & 0xFF
    f = bits & 0x7F
    if e == 0:
        return sign * math.ldexp(f, -126 - 7)
    return sign * math.ldexp(128 + f, e - 127 - 7)


def pin_torch_inputs(orc):
    """The tensors the GPU tests feed (torch bf16 on the CPU, int32 targets) reach
    the oracle as the exact numbers their bit patterns encode, and the head gives
    the same result for them as for those numbers given as fp64 arrays."""
    bits = [0x3F80, 0xC000, 0x0001, 0x007F, 0x0080, 0x7F7F, 0x3F81, 0x8000, 0xBEAA, 0x4B80, 0x3C23]
    t = torch.tensor(np.array(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
    got = orc._f64(t)
    assert got.dtype == np.float64
    want = np.array([_bf16_value(b) for b in bits])
    assert np.array_equal(got, want), (got, want)
    r = _rng(97)
    Xb = torch.tensor(r.integers(-2**15, 2**15, size=(5, 8)).astype(np.int16)).view(torch.bfloat16)
    Wb = torch.tensor(r.integers(-2**15, 2**15, size=(9, 8)).astype(np.int16)).view(torch.bfloat16)
    # keep finite, moderate values: clear the top exponent bits
    Xb = (Xb.view(torch.int16) & 0x3FFF).view(torch.bfloat16)
    Wb = (Wb.view(torch.int16) & 0x3FFF).view(torch.bfloat16)
    yt = torch.tensor([0, 8, IGN, 4, 2], dtype=torch.int32)
    dec = lambda a: np.vectorize(_bf16_value)(a.view(torch.int16).numpy().astype(np.uint16).astype(np.int64))  # noqa: E731
    l1, dX1, dW1, _, _ = orc.flce_reference(Xb, Wb, yt)
    l2, dX2, dW2, _, _ = orc.flce_reference(dec(Xb), dec(Wb), yt.numpy().astype(np.int64))
    assert l1 == l2 and np.array_equal(dX1, dX2) and np.array_equal(dW1, dW2)
    assert np.array_equal(orc._i64(yt), np.array([0, 8, IGN, 4, 2]))


def pin_reductions(orc):
    """'sum' is n times 'mean' (loss and both gradients); 'none' with per-row
    upstream weights g equals torch autograd of sum_i g_i * CE_i (reduction
    'none'), and its row losses equal torch's per-row cross-entropy."""
    X, W, y = _case(90, 13, 9, 21, n_ign=3)
    n = int((y != IGN).sum())
    lm, dXm, dWm, _, _ = orc.flce_reference(X, W, y, reduction="mean")
    ls, dXs, dWs, _, _ = orc.flce_reference(X, W, y, reduction="sum")
    assert abs(ls - n * lm) <= 1e-13 * abs(ls)
    _close(dXs, n * dXm, 1e-13, what="sum vs mean dX")
    _close(dWs, n * dWm, 1e-13, what="sum vs mean dW")
    g = _rng(91).standard_normal(13)
    ln, dXn, dWn, _, _, rows = orc.flce_reference(X, W, y, reduction="none", grad_row_scale=g, return_rows=True)
    tX = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    tW = torch.tensor(W, dtype=torch.float64, requires_grad=True)
    per_row = torch.nn.functional.cross_entropy(tX @ tW.T, torch.tensor(y), ignore_index=IGN, reduction="none")
    (per_row * torch.tensor(g)).sum().backward()
    _close(rows, per_row.detach().numpy(), 1e-12, what="row losses vs torch")
    assert abs(ln - float((per_row.detach() * torch.tensor(g)).sum())) <= 1e-12 * max(1.0, abs(ln))
    _close(dXn, tX.grad.numpy(), 1e-11, what="weighted dX vs autograd")
    _close(dWn, tW.grad.numpy(), 1e-11, what="weighted dW vs autograd")


def pin_ce_on_logits(orc):
    """Cross-entropy on given logits: torch's cross_entropy + autograd on the
    same fp64 logits for all three reductions, and the fused head's loss and
    dX = G W, dW = G^T X when the logits are X W^T."""
    r = _rng(100)
    Z = r.standard_normal((17, 40)) * 3.0
    y = r.integers(0, 40, size=17)
    y[[2, 9]] = IGN
    g = r.standard_normal(17)
    for red, w in (("mean", None), ("sum", None), ("none", g)):
        loss, dZ, lse, n, rows = orc.ce_reference(Z, y, reduction=red, grad_row_scale=w)
        tZ = torch.tensor(Z, requires_grad=True)
        per = torch.nn.functional.cross_entropy(tZ, torch.tensor(y), ignore_index=IGN, reduction="none")
        scale = {"mean": torch.full((17,), 1.0 / n, dtype=torch.float64), "sum": torch.ones(17, dtype=torch.float64),
                 "none": torch.tensor(g)}[red]
        tl = (per * scale).sum()
        tl.backward()
        assert abs(loss - tl.item()) <= 1e-12 * max(1.0, abs(tl.item())), (red, loss, tl.item())
        _close(dZ, tZ.grad.numpy(), 1e-12, atol=1e-16, what=f"dZ {red}")
        _close(rows, per.detach().numpy(), 1e-12, what=f"row losses {red}")
    X, W, yy = _case(101, 9, 6, 15, n_ign=2)
    l1, dX, dW, _, _ = orc.flce_reference(X, W, yy)
    l2, G, _, _, _ = orc.ce_reference(X @ W.T, yy)
    assert abs(l1 - l2) <= 1e-13 * abs(l1)
    _close(G @ W, dX, 1e-12, atol=1e-16, what="G W vs fused dX")
    _close(G.T @ X, dW, 1e-12, atol=1e-16, what="G^T X vs fused dW")


def pin_vocab_shards(orc):
    """Shard statistics and their merge: for a split of the vocabulary into
    uneven shards (one of a single entry, one holding no target), the merged
    log-sum-exp equals torch's logsumexp of the explicit fp64 logits, the merged
    target logit equals z[i, y_i], each shard's own log-sum-exp equals torch's
    over its columns, and ignored rows or targets outside a shard give 0."""
    X, W, y = _case(110, 11, 7, 37, n_ign=2)
    y[3] = 36  # the last vocabulary entry
    y[5] = 10  # the single-entry shard
    bounds = [0, 10, 11, 20, 37]
    y[(y >= 11) & (y < 20)] = 21  # shard [11, 20) holds no target
    Z = torch.tensor(X) @ torch.tensor(W).T
    lses, zys = [], []
    for v0, v1 in zip(bounds[:-1], bounds[1:]):
        lse_s, zy_s = orc.shard_stats(X, W[v0:v1], y, v0)
        _close(lse_s, torch.logsumexp(Z[:, v0:v1], dim=1).numpy(), 1e-13, what=f"shard lse [{v0},{v1})")
        inside = (y != IGN) & (y >= v0) & (y < v1)
        want = np.where(inside, Z.numpy()[np.arange(len(y)), np.where(inside, y, 0)], 0.0)
        assert np.array_equal(zy_s, want), f"shard target logits [{v0},{v1})"
        if v0 == 11:
            assert not np.any(zy_s), "a shard without targets reports none"
        lses.append(lse_s)
        zys.append(zy_s)
    lse, zy = orc.merge_shard_stats(np.stack(lses), np.stack(zys))
    _close(lse, torch.logsumexp(Z, dim=1).numpy(), 1e-13, what="merged lse")
    valid = y != IGN
    _close(zy[valid], Z.numpy()[np.arange(len(y))[valid], y[valid]], 1e-14, what="merged target logit")
    assert np.all(zy[~valid] == 0.0)
    per = torch.nn.functional.cross_entropy(Z, torch.tensor(y), ignore_index=IGN, reduction="none").numpy()
    _close(np.where(valid, lse - zy, 0.0), per, 1e-12, what="row losses from merged statistics")


def pin_pairwise_logistic(orc):
    """The DPO-form pair loss: torch's logsigmoid + autograd on the same
    sequence log-probabilities (a pair sharing a sequence with another pair
    included); one pair in closed form, log(1 + exp(-beta d)); swapping chosen
    and rejected turns softplus(-m) into softplus(m), whose difference is m."""
    r = _rng(120)
    lens = [5, 3, 7, 1, 4, 6]
    st = np.concatenate([[0], np.cumsum(lens)])
    N = int(st[-1])
    rl = np.abs(r.standard_normal(N)) * 3.0
    y = r.integers(0, 50, size=N)
    y[[0, 6, 9]] = IGN
    rl[y == IGN] = 0.0
    ch = np.array([0, 2, 4, 2])
    rj = np.array([1, 3, 5, 0])
    ref = r.standard_normal(6)
    beta = 0.7
    loss, logp, grad, w = orc.pairwise_logistic(rl, y, st, ch, rj, beta, ref)
    tl = torch.tensor(rl, requires_grad=True)
    tlogp = torch.stack([-tl[st[s]:st[s + 1]].sum() for s in range(6)])
    d = tlogp - torch.tensor(ref)
    tloss = -torch.nn.functional.logsigmoid(beta * (d[ch] - d[rj])).mean()
    tloss.backward()
    assert abs(loss - tloss.item()) <= 1e-13 * abs(tloss.item())
    _close(logp, tlogp.detach().numpy(), 1e-14, what="sequence log-probs")
    # the row weight is the upstream gradient of the row loss (valid rows only)
    want_w = np.where(y != IGN, tl.grad.numpy(), 0.0)
    _close(w, want_w, 1e-12, atol=1e-17, what="row weights vs autograd")
    rows_of = np.repeat(np.arange(6), lens)
    _close(-grad[rows_of][y != IGN], tl.grad.numpy()[y != IGN], 1e-12, what="dL/dlogp")
    # one pair: closed form
    one = np.array([0]), np.array([1])
    l1, lp1, g1, _ = orc.pairwise_logistic(rl, y, st, one[0], one[1], beta)
    dd = lp1[0] - lp1[1]
    assert abs(l1 - math.log1p(math.exp(-beta * dd))) <= 1e-13 * max(1.0, l1)
    assert abs(g1[0] + beta / (1.0 + math.exp(beta * dd))) <= 1e-13
    l2, _, _, _ = orc.pairwise_logistic(rl, y, st, one[1], one[0], beta)
    assert abs((l1 - l2) - (-beta * dd)) <= 1e-12 * max(1.0, abs(beta * dd))


ALL_PINS = [
    pin_zero_weight, pin_zero_input, pin_two_class, pin_large_logits,
    pin_torch_autograd, pin_finite_difference, pin_rows_of_g_sum_to_zero,
    pin_shift_invariance, pin_ignored_rows, pin_no_valid_rows, pin_target_range,
    pin_permutations, pin_equal_logits, pin_row_functions, pin_full_grads, pin_torch_inputs, pin_reductions,
    pin_ce_on_logits, pin_vocab_shards, pin_pairwise_logistic,
]
