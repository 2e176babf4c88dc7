"""Seeded random sweep of shapes and options, CUDA path against the fp64 oracle.

Each case draws N, H (a multiple of 8), V, an ignore pattern (scattered,
prompt-masked, both or none), a reduction (mean / sum / none with upstream
weights), per-row losses on or off and a workspace with or without the
packed-X area, so the whole-tile skip, the row reordering, ragged tiles and
chunk tails meet in combinations the hand-written cases do not list."""
import math

import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs
from oracle import flce_oracle as O
from test_parity_gpu import LOSS_RTOL, _lib, _np, assert_grad_close

pytestmark = pytest.mark.gpu

CASES = 24


def _draw(k):
    r = np.random.default_rng(1000 + k)
    N = int(r.integers(1, 1500))
    H = int(8 * r.integers(1, 65))            # 8 .. 512
    V = int(r.integers(2, 12000))
    pattern = ["none", "scattered", "prompt", "both"][int(r.integers(0, 4))]
    frac = float(r.uniform(0.05, 0.7)) if pattern in ("scattered", "both") else 0.0
    prefix = int(r.integers(1, N + 1)) if pattern in ("prompt", "both") and N > 1 else 0
    reduction = ["mean", "sum", "none"][int(r.integers(0, 3))]
    rows = bool(r.integers(0, 2))
    reorder = bool(r.integers(0, 2))
    return N, H, V, frac, prefix, reduction, rows, reorder


@pytest.mark.parametrize("k", range(CASES))
def test_random_case(k):
    F = _lib()
    N, H, V, frac, prefix, reduction, rows, reorder = _draw(k)
    w = custom(f"fuzz{k}", N=N, H=H, V=V, ignore_frac=frac, ignore_prefix=min(prefix, N))
    X, W, y = make_inputs(w)
    g = None
    kw = {}
    if reduction == "none":
        g = torch.randn(N, generator=torch.Generator().manual_seed(k)).float()
        kw["grad_row_scale"] = g.cuda()
    ws = F.alloc_workspace(N, H, V, reorder=reorder)
    loss, status, rl, dX, dW = F.forward_backward_ex(X.cuda(), W.cuda(), y.cuda(), reduction=reduction,
                                                    row_loss=rows, workspace=ws, **kw)
    torch.cuda.synchronize()
    assert status.item() == 0, (k, status.item())
    ref, rdX, rdW, _, n, ref_rows = O.flce_reference(X, W, y, reduction=reduction,
                                                     grad_row_scale=None if g is None else g.double().numpy(),
                                                     return_rows=True)
    scale = float(np.sum(np.abs(ref_rows * (g.double().numpy() if g is not None else 1.0))))
    if reduction == "mean":
        scale /= max(n, 1)
    assert abs(loss.item() - ref) <= LOSS_RTOL * max(scale, 1e-30) or (n == 0 and loss.item() == 0.0), \
        (k, loss.item(), ref)
    assert_grad_close(_np(dX), rdX, f"dX case {k}")
    assert_grad_close(_np(dW), rdW, f"dW case {k}")
    assert torch.count_nonzero(dX[(y == -100).cuda()]).item() == 0
    if rows:
        got = rl.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(got - ref_rows)) <= LOSS_RTOL * max(1.0, np.max(np.abs(ref_rows))), k
    reordered, n_valid = F.row_order_info(ws)
    assert n_valid == n
    if reordered:
        v = (y != -100).numpy().astype(np.int64)
        tiles = np.add.reduceat(v, np.arange(0, N, 256))
        assert reorder and math.ceil(n / 256) < int((tiles > 0).sum())
