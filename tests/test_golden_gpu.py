"""The guide's worked example of the fused loss (configuration in
tests/golden/guide_flce_example.json, cited there): hidden 4096, vocabulary
128256, 1024 token rows, standard-normal X and W in bf16, uniform labels.  The
page prints no value, so the head is checked against the oracle: the loss over
every row exactly, dX and dW on sampled rows."""
import json
import os

import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs
from oracle import flce_oracle as O
from test_parity_full_gpu import _sample_rows
from test_parity_gpu import assert_grad_close, assert_loss_close

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "guide_flce_example.json")


def test_guide_example_configuration():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    g = json.load(open(GOLDEN))
    w = custom("guide_example", N=g["batch_seq"], H=g["hidden_size"], V=g["vocab_size"], x_std=g["x_std"],
               w_std=g["w_std"])
    X, W, y = make_inputs(w)
    loss, dX, dW = F.forward_backward(X.cuda(), W.cuda(), y.cuda())
    torch.cuda.synchronize()
    y_np = y.numpy().astype(np.int64)
    rows, vrows = _sample_rows(y_np, w.N, w.V, np.random.default_rng(7))
    gX = dX[torch.as_tensor(rows, device="cuda")].float().cpu().numpy().astype(np.float64)
    gW = dW[torch.as_tensor(vrows, device="cuda")].float().cpu().numpy().astype(np.float64)
    W64 = W.float().numpy().astype(np.float64)
    X64 = X.float().numpy().astype(np.float64)
    ref_loss, lse, n = O.full_loss(X64, W64, y_np, W64=W64)
    assert n == w.N
    assert ref_loss > 100.0  # logits of standard deviation 64: far from ln V
    assert_loss_close(loss, ref_loss)
    assert_grad_close(gX, O.dx_rows(X64, W64, y_np, rows, lse[rows], n, W64=W64), "dX sampled rows")
    assert_grad_close(gW, O.dw_rows(X64, W64, y_np, vrows, lse, n, W64=W64, X64=X64), "dW sampled rows")
