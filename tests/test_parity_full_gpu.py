"""Full-size workloads, in the launch configuration the benchmark times.

The oracle cannot hold N x V fp64 logits at these sizes, so it evaluates its
per-row definition: the loss over every row exactly (all N log-sum-exps), dX on
sampled token rows and dW on sampled vocabulary rows (including the targets that
occur most often, the chunk boundaries and the last vocabulary row).
"""
import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.inputs import WORKLOADS, make_inputs
from oracle import flce_oracle as O
from test_parity_gpu import assert_grad_close, assert_loss_close

pytestmark = pytest.mark.gpu

FULL = ["llama3_8b_head", "long_context", "gemma2_large_vocab", "phi3_mini_small_vocab"]


def _sample_rows(y, N, V, rng):
    yv = y[y != -100]
    tok = set(rng.choice(N, size=48, replace=False).tolist()) | {0, N - 1, N // 2}
    ign = np.nonzero(y == -100)[0]
    if len(ign):
        tok |= set(rng.choice(ign, size=min(8, len(ign)), replace=False).tolist())
    vals, counts = np.unique(yv, return_counts=True)
    hot = vals[np.argsort(-counts)[:8]]
    voc = set(rng.choice(V, size=40, replace=False).tolist()) | set(hot.tolist())
    voc |= {0, V - 1, min(2047, V - 1), min(2048, V - 1), min(4095, V - 1)}
    return np.array(sorted(tok)), np.array(sorted(voc))


@pytest.mark.parametrize("name", FULL)
def test_full_size_against_oracle(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    F.load_library()
    w = WORKLOADS[name]
    X, W, y = make_inputs(w)
    loss, dX, dW = F.forward_backward(X.cuda(), W.cuda(), y.cuda())
    torch.cuda.synchronize()
    y_np = y.numpy().astype(np.int64)
    rng = np.random.default_rng(1234)
    rows, vrows = _sample_rows(y_np, w.N, w.V, rng)
    gX = dX[torch.as_tensor(rows, device="cuda")].float().cpu().numpy().astype(np.float64)
    gW = dW[torch.as_tensor(vrows, device="cuda")].float().cpu().numpy().astype(np.float64)
    del dX, dW
    torch.cuda.empty_cache()

    W64 = W.float().numpy().astype(np.float64)
    X64 = X.float().numpy().astype(np.float64)
    ref_loss, lse, n = O.full_loss(X64, W64, y_np, W64=W64)
    assert n == w.N - w.n_ignored
    assert_loss_close(loss, ref_loss)
    ref_dX = O.dx_rows(X64, W64, y_np, rows, lse[rows], n, W64=W64)
    assert_grad_close(gX, ref_dX, f"{name} dX sampled rows")
    ign = y_np[rows] == -100
    assert np.all(gX[ign] == 0.0)
    ref_dW = O.dw_rows(X64, W64, y_np, vrows, lse, n, W64=W64, X64=X64)
    assert_grad_close(gW, ref_dW, f"{name} dW sampled rows")
