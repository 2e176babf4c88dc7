"""Cross-entropy on given logits (the unfused counterpart of the head) against
the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import flce_oracle as O
from test_parity_gpu import LOSS_RTOL, assert_grad_close, assert_loss_close

pytestmark = pytest.mark.gpu


def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    F.load_library()
    return F


def _case(N, V, std=1.28, ign=0.1, seed=0):
    g = torch.Generator().manual_seed(seed)
    Z = (torch.randn(N, V, generator=g) * std).to(torch.bfloat16)
    y = torch.randint(0, V, (N,), generator=g, dtype=torch.int64).to(torch.int32)
    k = int(ign * N)
    if k:
        y[torch.randperm(N, generator=g)[:k]] = -100
    return Z, y


def _check(Z, y, reduction="mean", grad_row_scale=None, grad="new"):
    F = _lib()
    Zd = Z.cuda()
    w = None if grad_row_scale is None else torch.as_tensor(grad_row_scale, dtype=torch.float32).cuda()
    loss, status, rl, dz = F.cross_entropy(Zd, y.cuda(), reduction=reduction, grad_row_scale=w, row_loss=True,
                                           grad=grad)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref, rdz, _, _, rows = O.ce_reference(Z, y, reduction=reduction,
                                          grad_row_scale=None if w is None else np.asarray(grad_row_scale))
    assert_loss_close(loss.item(), ref)
    r = rl.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(r - rows)) <= LOSS_RTOL * max(np.max(np.abs(rows)), 1e-30)
    if dz is not None:
        assert_grad_close(dz.float().cpu().numpy().astype(np.float64), rdz, "dlogits")
    return dz


# Widths with V % 8 == 0 take the 16-byte vector path, others the scalar one.
@pytest.mark.parametrize("N,V", [(256, 4096), (300, 5000), (1, 300), (129, 100), (64, 1001), (17, 3),
                                 (9, 40000), (5, 200000), (3, 300000)])
def test_ce_small(N, V):
    Z, y = _case(N, V)
    _check(Z, y)


def test_ce_reductions_and_weights():
    Z, y = _case(200, 3000)
    _check(Z, y, reduction="sum")
    g = np.random.default_rng(3).standard_normal(200)
    _check(Z, y, reduction="none", grad_row_scale=g)


def test_ce_in_place_and_forward_only():
    F = _lib()
    Z, y = _case(257, 6000)
    ref = _check(Z, y)
    Zd = Z.cuda()
    F.cross_entropy(Zd, y.cuda(), grad="inplace")
    torch.cuda.synchronize()
    assert torch.equal(Zd, ref)
    loss, status, rl, dz = F.cross_entropy(Z.cuda(), y.cuda(), grad="none")
    torch.cuda.synchronize()
    assert dz is None and status.item() == 0
    assert_loss_close(loss.item(), O.ce_reference(Z, y)[0])


def test_ce_large_logits_and_all_ignored():
    Z, y = _case(128, 2048, std=30.0)
    _check(Z, y)
    y[:] = -100
    dz = _check(Z, y)
    assert torch.count_nonzero(dz).item() == 0


def test_ce_target_out_of_range():
    F = _lib()
    Z, y = _case(64, 500, ign=0)
    y[5] = 500
    _, status, _, _ = F.cross_entropy(Z.cuda(), y.cuda())
    torch.cuda.synchronize()
    assert status.item() == 4


def test_ce_full_size_llama_logits():
    """N = 8192 tokens x V = 128256 (2.1 GB of logits): the loss against the
    oracle over every row (row blocks), dlogits on sampled rows."""
    F = _lib()
    N, V = 8192, 128256
    Z, y = _case(N, V, ign=0.05, seed=1)
    loss, status, rl, dz = F.cross_entropy(Z.cuda(), y.cuda(), row_loss=True)
    torch.cuda.synchronize()
    assert status.item() == 0
    n = int((y != -100).sum())
    total = 0.0
    rows_ref = np.empty(N)
    for b in range(0, N, 512):
        l, _, _, _, rows = O.ce_reference(Z[b:b + 512], y[b:b + 512], reduction="sum")
        total += l
        rows_ref[b:b + 512] = rows
    assert_loss_close(loss.item(), total / n)
    r = rl.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(r - rows_ref)) <= LOSS_RTOL * np.max(np.abs(rows_ref))
    pick = np.array([0, 1, 777, 4096, 8191])
    _, rdz, _, _, _ = O.ce_reference(Z[pick], y[pick], reduction="none", grad_row_scale=np.full(len(pick), 1.0 / n))
    assert_grad_close(dz[torch.as_tensor(pick).cuda()].float().cpu().numpy().astype(np.float64), rdz, "dlogits rows")
