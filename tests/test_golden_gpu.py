"""The guide's worked example of the fused loss (configuration in
tests/golden/guide_flce_example.json, cited there): hidden 4096, vocabulary
128256, 1024 token rows, standard-normal X and W in bf16, uniform labels.  The
page prints no value, so the head is checked against the oracle: the loss and
every element of dX and dW."""
import json
import os

import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs
from test_parity_full_gpu import check_against_full_oracle

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
    dX_cpu, dW_cpu = dX.cpu(), dW.cpu()
    del dX, dW
    ref_loss = check_against_full_oracle(X, W, y, loss, dX_cpu, dW_cpu, "guide example", n_expected=w.N)
    assert ref_loss > 100.0  # logits of standard deviation 64: far from ln V
