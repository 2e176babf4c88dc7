"""Fused-linear preference loss (pairwise logistic, DPO form) on top of the
head: the glue on CPU with the fp64 oracle standing in for the two head calls,
and the CUDA path on the GPU; both against torch fp64 autograd through explicit
logits, log-softmax and per-sequence sums."""
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
    seq = torch.cat([torch.full((n,), s, dtype=torch.int64) for s, n in enumerate(lens)])
    start = 0
    for n in lens:
        y[start:start + prompt] = -100
        start += n
    chosen = torch.tensor([0, 2, 4])
    rejected = torch.tensor([1, 3, 5])
    ref = torch.randn(len(lens), generator=g, dtype=torch.float64) * 3.0
    return X, W, y, seq, chosen, rejected, ref


def _autograd_reference(X, W, y, seq, chosen, rejected, beta, ref):
    Xt = X.double().clone().requires_grad_(True)
    Wt = W.double().clone().requires_grad_(True)
    logsm = torch.log_softmax(Xt @ Wt.T, dim=1)
    valid = y != -100
    tok = torch.where(valid, logsm.gather(1, torch.where(valid, y, 0).long()[:, None])[:, 0], torch.zeros(()))
    logp = torch.zeros(int(seq.max()) + 1, dtype=torch.float64).index_add(0, seq, tok)
    d = logp - ref
    loss = -torch.nn.functional.logsigmoid(beta * (d[chosen] - d[rejected])).mean()
    loss.backward()
    return loss.item(), Xt.grad.numpy(), Wt.grad.numpy(), logp.detach().numpy()


def _oracle_rows(X, W, y, ignore_index):
    _, _, _, _, _, rows = O.flce_reference(X, W, y, ignore_index, reduction="none", return_rows=True)
    return torch.tensor(rows), torch.zeros(1, dtype=torch.int32)


def _oracle_grads(X, W, y, ignore_index, weights):
    _, dX, dW, _, _ = O.flce_reference(X, W, y, ignore_index, reduction="none", grad_row_scale=weights.double().numpy())
    return torch.tensor(dX), torch.tensor(dW), torch.zeros(1, dtype=torch.int32)


def test_preference_glue_with_oracle_head():
    X, W, y, seq, chosen, rejected, ref = _packed()
    beta = 0.5
    loss, dX, dW, logp = preference_forward_backward(X, W, y, seq, chosen, rejected, beta, ref,
                                                     head_rows=_oracle_rows, head_grads=_oracle_grads)
    rl, rdX, rdW, rlogp = _autograd_reference(X, W, y, seq, chosen, rejected, beta, ref)
    np.testing.assert_allclose(logp.numpy(), rlogp, rtol=1e-12)
    assert abs(loss.item() - rl) <= 1e-12 * abs(rl)
    # the fp32 upstream weights set the precision of the gradients
    np.testing.assert_allclose(dX.numpy(), rdX, rtol=1e-6, atol=1e-9 * np.abs(rdX).max())
    np.testing.assert_allclose(dW.numpy(), rdW, rtol=1e-6, atol=1e-9 * np.abs(rdW).max())


@pytest.mark.gpu
def test_preference_on_the_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_parity_gpu import assert_grad_close
    X, W, y, seq, chosen, rejected, ref = _packed(seed=1, H=256, V=5000, lens=(300, 280, 410, 256, 333, 297),
                                                  prompt=60)
    beta = 0.005  # margins of order one: sequence log-probs here are in the thousands
    loss, dX, dW, logp = preference_forward_backward(X.cuda(), W.cuda(), y.cuda(), seq.cuda(), chosen.cuda(),
                                                     rejected.cuda(), beta, ref.cuda())
    rl, rdX, rdW, rlogp = _autograd_reference(X, W, y, seq, chosen, rejected, beta, ref)
    got = logp.cpu().numpy()
    assert np.max(np.abs(got - rlogp)) <= 1e-4 * np.max(np.abs(rlogp))
    assert abs(loss.item() - rl) <= 1e-3 * abs(rl)
    assert_grad_close(dX.float().cpu().numpy(), rdX, "dX")
    assert_grad_close(dW.float().cpu().numpy(), rdW, "dW")
