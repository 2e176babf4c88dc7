"""Fused-linear preference loss (pairwise logistic, DPO form) on top of the
head: the glue on CPU with the fp64 oracle standing in for the library's three
calls, and the CUDA path on the GPU; both against torch fp64 autograd through
explicit logits, log-softmax and per-sequence sums.  The library's pair-loss
step alone is checked against the oracle's on the GPU."""
import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.preference import preference_forward_backward
from oracle import flce_oracle as O


def _packed(seed=0, H=32, V=300, lens=(40, 37, 52, 29, 33, 45), prompt=8):
    """Six sequences (three pairs) packed as token rows; the first `prompt`
    rows of each sequence are ignored (prompt tokens)."""
    g = torch.Generator().manual_seed(seed)
    N = sum(lens)
    X = torch.randn(N, H, generator=g).to(torch.bfloat16)
    W = (torch.randn(V, H, generator=g) * 0.2).to(torch.bfloat16)
    y = torch.randint(0, V, (N,), generator=g, dtype=torch.int32)
    seq_start = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    for s in range(len(lens)):
        y[seq_start[s]:seq_start[s] + prompt] = -100
    chosen = torch.tensor([0, 2, 4], dtype=torch.int32)
    rejected = torch.tensor([1, 3, 5], dtype=torch.int32)
    ref = torch.randn(len(lens), generator=g, dtype=torch.float64) * 3.0
    return X, W, y, seq_start, chosen, rejected, ref


def _autograd_reference(X, W, y, seq_start, chosen, rejected, beta, ref):
    lens = (seq_start[1:] - seq_start[:-1]).long()
    seq = torch.repeat_interleave(torch.arange(len(lens)), lens)
    Xt = X.double().clone().requires_grad_(True)
    Wt = W.double().clone().requires_grad_(True)
    logsm = torch.log_softmax(Xt @ Wt.T, dim=1)
    valid = y != -100
    tok = torch.where(valid, logsm.gather(1, torch.where(valid, y, 0).long()[:, None])[:, 0], torch.zeros(()))
    logp = torch.zeros(len(lens), dtype=torch.float64).index_add(0, seq, tok)
    d = logp - ref
    loss = -torch.nn.functional.logsigmoid(beta * (d[chosen.long()] - d[rejected.long()])).mean()
    loss.backward()
    return loss.item(), Xt.grad.numpy(), Wt.grad.numpy(), logp.detach().numpy()


def _oracle_rows(X, W, y, ignore_index):
    _, _, _, _, _, rows = O.flce_reference(X, W, y, ignore_index, reduction="none", return_rows=True)
    return torch.tensor(rows), torch.zeros(1, dtype=torch.int32)


def _oracle_pair(row_loss, y, seq_start, chosen, rejected, beta, ref, ignore_index):
    loss, logp, grad, w = O.pairwise_logistic(row_loss, y, seq_start, chosen, rejected, beta, ref, ignore_index)
    return (torch.tensor([loss], dtype=torch.float64), torch.tensor(logp), torch.tensor(grad), torch.tensor(w, dtype=torch.float32),
            torch.zeros(1, dtype=torch.int32))


def _oracle_grads(X, W, y, ignore_index, weights):
    _, dX, dW, _, _ = O.flce_reference(X, W, y, ignore_index, reduction="none", grad_row_scale=weights.double().numpy())
    return torch.tensor(dX), torch.tensor(dW), torch.zeros(1, dtype=torch.int32)


def test_preference_glue_with_oracle_steps():
    X, W, y, st, chosen, rejected, ref = _packed()
    beta = 0.5
    loss, dX, dW, logp = preference_forward_backward(X, W, y, st, chosen, rejected, beta, ref,
                                                     head_rows=_oracle_rows, pair_loss=_oracle_pair,
                                                     head_grads=_oracle_grads)
    rl, rdX, rdW, rlogp = _autograd_reference(X, W, y, st, chosen, rejected, beta, ref)
    np.testing.assert_allclose(logp.numpy(), rlogp, rtol=1e-12)
    assert abs(loss.item() - rl) <= 1e-12 * abs(rl)
    # the fp32 upstream weights set the precision of the gradients
    np.testing.assert_allclose(dX.numpy(), rdX, rtol=1e-6, atol=1e-9 * np.abs(rdX).max())
    np.testing.assert_allclose(dW.numpy(), rdW, rtol=1e-6, atol=1e-9 * np.abs(rdW).max())


def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    F.load_library()
    return F


@pytest.mark.gpu
def test_preference_on_the_gpu():
    _lib()
    from test_parity_gpu import assert_grad_close
    X, W, y, st, chosen, rejected, ref = _packed(seed=1, H=256, V=5000, lens=(300, 280, 410, 256, 333, 297),
                                                 prompt=60)
    beta = 0.005  # margins of order one: sequence log-probs here are in the thousands
    loss, dX, dW, logp = preference_forward_backward(X.cuda(), W.cuda(), y.cuda(), st.cuda(), chosen.cuda(),
                                                     rejected.cuda(), beta, ref.cuda())
    rl, rdX, rdW, rlogp = _autograd_reference(X, W, y, st, chosen, rejected, beta, ref)
    got = logp.cpu().numpy()
    assert np.max(np.abs(got - rlogp)) <= 1e-4 * np.max(np.abs(rlogp))
    assert abs(loss.item() - rl) <= 1e-3 * abs(rl)
    assert_grad_close(dX.float().cpu().numpy(), rdX, "dX")
    assert_grad_close(dW.float().cpu().numpy(), rdW, "dW")


@pytest.mark.gpu
@pytest.mark.parametrize("S,P,shared,with_ref", [(6, 3, False, True), (40, 70, True, False), (1000, 600, True, True)])
def test_pair_loss_step_against_oracle(S, P, shared, with_ref):
    """flce_pairwise_logistic on given row losses: the loss, the sequence
    log-probabilities, their gradient and the rows' weights against the
    oracle (pairs may share sequences; empty sequences allowed)."""
    F = _lib()
    r = np.random.default_rng(S + P)
    lens = r.integers(0, 30, size=S)
    st = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    N = int(st[-1]) + 5  # rows past the last sequence belong to none
    y = r.integers(0, 100, size=N).astype(np.int32)
    y[r.random(N) < 0.2] = -100
    rl = np.where(y != -100, np.abs(r.standard_normal(N)) * 4.0, 0.0).astype(np.float32)
    if shared:
        ch = r.integers(0, S, size=P).astype(np.int32)
        rj = r.integers(0, S, size=P).astype(np.int32)
    else:
        ch = np.arange(0, 2 * P, 2, dtype=np.int32)
        rj = ch + 1
    ref = r.standard_normal(S) if with_ref else None
    beta = 0.3
    t = lambda a: None if a is None else torch.tensor(a).cuda()  # noqa: E731
    loss, logp, grad, w, status = F.pairwise_logistic(t(rl), t(y), t(st), t(ch), t(rj), beta, t(ref))
    torch.cuda.synchronize()
    assert status.item() == 0
    rl_, rlogp, rgrad, rw = O.pairwise_logistic(rl, y, st, ch, rj, beta, ref)
    assert abs(loss.item() - rl_) <= 1e-12 * max(1.0, abs(rl_))
    np.testing.assert_allclose(logp.cpu().numpy(), rlogp, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(grad.cpu().numpy(), rgrad, rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-12)
    # the same inputs again: bit-identical (fixed-order sums)
    loss2, logp2, grad2, w2, _ = F.pairwise_logistic(t(rl), t(y), t(st), t(ch), t(rj), beta, t(ref))
    assert loss2.item() == loss.item() and torch.equal(grad2, grad) and torch.equal(w2, w)


@pytest.mark.gpu
def test_pair_loss_step_reports_bad_ids():
    F = _lib()
    rl = torch.ones(10, device="cuda")
    y = torch.zeros(10, dtype=torch.int32, device="cuda")
    st = torch.tensor([0, 4, 10], dtype=torch.int32, device="cuda")
    ch = torch.tensor([0], dtype=torch.int32, device="cuda")
    for rj, st_ in ((torch.tensor([2], dtype=torch.int32, device="cuda"), st),  # sequence id past S
                    (torch.tensor([1], dtype=torch.int32, device="cuda"),
                     torch.tensor([0, 4, 11], dtype=torch.int32, device="cuda"))):  # rows past N
        *_, status = F.pairwise_logistic(rl, y, st_, ch, rj, 0.1)
        torch.cuda.synchronize()
        assert status.item() == 1  # FLCE_ERR_INVALID_ARGUMENT
