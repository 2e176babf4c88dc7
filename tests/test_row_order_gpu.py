"""Scattered ignored targets: the token rows are reordered on the device (valid
rows first, a stable partition), X is packed in that order and dX and the
per-row losses go back to the caller's rows.  CUDA path against the fp64 oracle, with
the same tolerances as the other parity tests, plus a check that the call
really took (or did not take) the reordered path."""
import math

import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs
from oracle import flce_oracle as O
from test_parity_gpu import LOSS_RTOL, _lib, _np, assert_grad_close, assert_loss_close

pytestmark = pytest.mark.gpu


def expect_reorder(y, ignore_index=-100):
    """The library's rule: reorder when the valid rows, packed first, fill fewer
    256-row tiles than the tiles that hold any valid row."""
    v = (y != ignore_index).numpy().astype(np.int64)
    tiles = np.add.reduceat(v, np.arange(0, len(v), 256))
    return math.ceil(int(v.sum()) / 256) < int((tiles > 0).sum())


def _call(X, W, y, reorder=True, **kw):
    F = _lib()
    # small cases: the packed-X area exceeds 5% of their logits, so ask for it
    ws = F.alloc_workspace(X.shape[0], X.shape[1], W.shape[0], reorder=reorder)
    loss, status, rl, dX, dW = F.forward_backward_ex(X.cuda(), W.cuda(), y.cuda(), workspace=ws, **kw)
    torch.cuda.synchronize()
    assert status.item() == 0
    reordered, n_valid = F.row_order_info(ws)
    assert n_valid == int((y != -100).sum())
    return loss.item(), rl, dX, dW, reordered


SCATTERED = [
    custom("scattered_half", N=1536, H=256, V=5000, ignore_frac=0.5),        # 768 valid rows: 3 tiles, not 6
    custom("scattered_ragged", N=1000, H=136, V=6208, ignore_frac=0.3),      # ragged N and V, 3 of 4 tiles
    custom("scattered_long_k", N=700, H=4096, V=1200, ignore_frac=0.4),      # one chunk, H = 64 k-blocks
    custom("scattered_zipf", N=2100, H=320, V=9000, targets="zipf", ignore_frac=0.35),
    custom("scattered_most", N=1300, H=64, V=3000, ignore_frac=0.9),         # 130 valid rows in one tile
]


@pytest.mark.parametrize("w", SCATTERED, ids=lambda w: w.name)
def test_scattered_ignores_reordered(w):
    X, W, y = make_inputs(w)
    assert expect_reorder(y)
    loss, _, dX, dW, reordered = _call(X, W, y)
    assert reordered
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(loss, rl)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")
    assert torch.count_nonzero(dX[(y == -100).cuda()]).item() == 0


def test_prompt_mask_and_scattered_ignores():
    """Whole ignored tiles and scattered ignores together."""
    w = custom("prompt_and_scattered", N=1800, H=192, V=4500, ignore_prefix=520, ignore_frac=0.2)
    X, W, y = make_inputs(w)
    assert expect_reorder(y)
    loss, _, dX, dW, reordered = _call(X, W, y)
    assert reordered
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(loss, rl)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")


@pytest.mark.parametrize("case", ["all_valid", "aligned_prompt_mask", "sparse_ignores"])
def test_no_reorder_when_it_saves_no_tile(case):
    w = custom(f"keep_{case}", N=1024, H=128, V=3000, ignore_frac=0.02 if case == "sparse_ignores" else 0.0)
    X, W, y = make_inputs(w)
    if case == "aligned_prompt_mask":
        y[:512] = -100
    assert not expect_reorder(y)
    loss, _, dX, dW, reordered = _call(X, W, y)
    assert not reordered
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(loss, rl)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")


def test_reordered_reduction_none_rows_back_in_place():
    """Upstream weights and per-row losses follow the caller's row order."""
    w = custom("reorder_none", N=1100, H=264, V=5000, ignore_frac=0.45)
    g = torch.randn(1100, generator=torch.Generator().manual_seed(9)).float()
    X, W, y = make_inputs(w)
    assert expect_reorder(y)
    loss, rl, dX, dW, reordered = _call(X, W, y, reduction="none", grad_row_scale=g.cuda(), row_loss=True)
    assert reordered
    ref, rdX, rdW, _, _, rows = O.flce_reference(X, W, y, reduction="none", grad_row_scale=g.double().numpy(),
                                                 return_rows=True)
    assert abs(loss - ref) <= LOSS_RTOL * float(np.sum(np.abs(g.double().numpy() * rows)))
    assert_grad_close(_np(dX), rdX, "dX none")
    assert_grad_close(_np(dW), rdW, "dW none")
    r = rl.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(r - rows)) <= LOSS_RTOL * np.max(np.abs(rows))
    assert np.all(r[y.numpy() == -100] == 0.0)


def test_reordered_forward_only():
    w = custom("reorder_fwd", N=900, H=128, V=4000, ignore_frac=0.5)
    X, W, y = make_inputs(w)
    assert expect_reorder(y)
    loss, rl, dX, dW, reordered = _call(X, W, y, grads=False, row_loss=True)
    assert reordered and dX is None and dW is None
    ref, _, _, _, _, rows = O.flce_reference(X, W, y, return_rows=True)
    assert_loss_close(loss, ref)
    r = rl.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(r - rows)) <= LOSS_RTOL * np.max(np.abs(rows))


def test_reordered_mean_over_external_count():
    w = custom("reorder_count", N=800, H=136, V=3000, ignore_frac=0.5)
    X, W, y = make_inputs(w)
    count = 2000
    loss, _, dX, dW, reordered = _call(X, W, y, mean_count=torch.tensor([count], dtype=torch.int32).cuda())
    assert reordered
    valid = (y != -100).numpy()
    ref, rdX, rdW, _, _ = O.flce_reference(X, W, y, reduction="none", grad_row_scale=np.where(valid, 1.0 / count, 0.0))
    assert_loss_close(loss, ref)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")


def test_reordered_repeat_calls_identical():
    F = _lib()
    w = custom("reorder_repeat", N=1536, H=256, V=5000, ignore_frac=0.5)
    X, W, y = (t.cuda() for t in make_inputs(w))
    a = F.forward_backward(X, W, y)
    b = F.forward_backward(X, W, y)
    assert a[0] == b[0]
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_base_workspace_keeps_the_order():
    """Without the packed-X area the rows keep their order; results are the same."""
    w = custom("base_ws", N=1536, H=256, V=5000, ignore_frac=0.5)
    X, W, y = make_inputs(w)
    assert expect_reorder(y)
    loss, _, dX, dW, reordered = _call(X, W, y, reorder=False)
    assert not reordered
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(loss, rl)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")


def test_benchmark_workspace_reorders_the_large_vocab_shape():
    """At the Gemma-2-like shape the packed-X area fits the 5% budget, so the
    workspace the benchmark gives it reorders its scattered ignores (its
    full-size parity against the oracle is in test_parity_full_gpu)."""
    F = _lib()
    from lm_head_linear_03_b200.inputs import WORKLOADS
    w = WORKLOADS["gemma2_large_vocab"]
    X, W, y = make_inputs(w, "cuda")
    assert F.reorder_fits(w.N, w.H, w.V)
    ws = F.alloc_workspace(w.N, w.H, w.V, reorder=True)
    assert ws.numel() == F.workspace_size_reorder(w.N, w.H) > F.workspace_size(w.N, w.H, w.V)
    loss, status, _, dX, dW = F.forward_backward_ex(X, W, y, workspace=ws)
    torch.cuda.synchronize()
    assert status.item() == 0
    reordered, n_valid = F.row_order_info(ws)
    assert reordered and n_valid == int((y != -100).sum())
    assert torch.count_nonzero(dX[y == -100]).item() == 0


def test_host_entry_with_reordered_rows():
    """The host-buffer entry (W in pieces, pass 2 in sections) on reordered rows:
    packed X, dX scattered back, both copied out; checked against the oracle."""
    F = _lib()
    w = custom("host_reorder", N=1300, H=256, V=7000, ignore_frac=0.4)
    X, W, y = make_inputs(w)
    assert expect_reorder(y)
    hX, hW, hy = X.pin_memory(), W.pin_memory(), y.pin_memory()
    ws = F.alloc_workspace(w.N, w.H, w.V, reorder=True)
    dev = (torch.empty_like(X, device="cuda"), torch.empty_like(W, device="cuda"),
           torch.empty_like(y, device="cuda"), torch.empty_like(X, device="cuda"),
           torch.empty_like(W, device="cuda"), ws)
    loss, hdX, hdW = F.forward_backward_host(hX, hW, hy, dev)
    reordered, _ = F.row_order_info(ws)
    assert reordered
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(loss, rl)
    assert_grad_close(_np(hdX), rdX, "dX")
    assert_grad_close(_np(hdW), rdW, "dW")
    assert torch.count_nonzero(hdX[y == -100]).item() == 0
