"""Full-size workloads, in the launch configuration the benchmark times.

Every element of the loss, dX and dW is compared with the fp64 oracle.  The
oracle cannot hold N x V fp64 logits at these sizes, so it takes the rows a
block at a time (``full_grads``): the same definition, with only one block's
logits in memory.  That is minutes of host fp64 per workload on a many-core
host.
"""
import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.inputs import WORKLOADS, make_inputs
from oracle import flce_oracle as O
from test_parity_gpu import FRO_RTOL, MAXABS_FRAC, assert_loss_close

pytestmark = pytest.mark.gpu

FULL = ["llama3_8b_head", "long_context", "gemma2_large_vocab", "phi3_mini_small_vocab"]


def assert_grad_close_blocked(got, ref, what, block=4096):
    """The parity tolerances (relative Frobenius error <= 1e-2, max-abs error <=
    2^-7 * max|ref|) over every element of ``got`` (a bf16 CPU tensor) against
    ``ref`` (fp64), taken a block of rows at a time to bound host memory."""
    assert tuple(got.shape) == ref.shape, (what, tuple(got.shape), ref.shape)
    num = den = 0.0
    max_err = max_ref = 0.0
    for r0 in range(0, ref.shape[0], block):
        g = got[r0:r0 + block].float().numpy().astype(np.float64)
        r = ref[r0:r0 + block]
        d = g - r
        num += float(np.sum(d * d))
        den += float(np.sum(r * r))
        max_err = max(max_err, float(np.max(np.abs(d))))
        max_ref = max(max_ref, float(np.max(np.abs(r))))
    if den == 0.0:
        assert num == 0.0, f"{what}: expected exact zeros"
        return
    fro = (num / den) ** 0.5
    assert fro <= FRO_RTOL, f"{what}: relative Frobenius error {fro:.3e}"
    assert max_err <= MAXABS_FRAC * max_ref, f"{what}: max-abs error {max_err:.3e} > {MAXABS_FRAC * max_ref:.3e}"
    return fro, max_err / max_ref


def check_against_full_oracle(X, W, y, loss, dX_cpu, dW_cpu, what, n_expected=None):
    """Loss, every dX row and every dW row of one call against ``full_grads``;
    returns the oracle's loss."""
    y_np = y.numpy().astype(np.int64)
    X64 = X.float().numpy().astype(np.float64)
    W64 = W.float().numpy().astype(np.float64)
    ref_loss, rdX, rdW, _, n = O.full_grads(X64, W64, y_np, W64=W64, X64=X64)
    del W64
    if n_expected is not None:
        assert n == n_expected
    assert_loss_close(loss, ref_loss)
    ign = torch.as_tensor(y_np == -100)
    assert not dX_cpu[ign].float().any(), f"{what}: ignored rows of dX are not zero"
    assert_grad_close_blocked(dX_cpu, rdX, f"{what} dX")
    del rdX
    assert_grad_close_blocked(dW_cpu, rdW, f"{what} dW")
    return ref_loss


@pytest.mark.parametrize("name", FULL)
def test_full_size_against_oracle(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    F.load_library()
    w = WORKLOADS[name]
    X, W, y = make_inputs(w)
    # the benchmark's launch: the async entry on the workspace it chooses
    ws = F.alloc_workspace(w.N, w.H, w.V, reorder=F.reorder_fits(w.N, w.H, w.V))
    loss_t, status, dX, dW = F.forward_backward_async(X.cuda(), W.cuda(), y.cuda(), workspace=ws)
    torch.cuda.synchronize()
    assert status.item() == 0
    loss = loss_t.item()
    dX_cpu, dW_cpu = dX.cpu(), dW.cpu()
    del dX, dW, ws
    torch.cuda.empty_cache()
    check_against_full_oracle(X, W, y, loss, dX_cpu, dW_cpu, name, n_expected=w.N - w.n_ignored)
