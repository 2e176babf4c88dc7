"""The allocation-free entry point against the ordinary workspace entry point.

flce_forward_backward_noalloc is for callers that cannot allocate device
memory: a plug-in that is only handed its tensors, or a process whose
framework pool already holds nearly all of the GPU.  It takes its scratch from
a fixed array inside the library instead of a caller-provided workspace, and
every call reuses that array, so two calls in a row must each agree with the
workspace entry on the same inputs.
"""
import ctypes

import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs
from test_parity_gpu import assert_grad_close, assert_loss_close


def _np(t):
    return t.float().cpu().numpy()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    from lm_head_linear_03_b200 import flce
    F.load_library()
    cases = [custom("noalloc_a", N=300, H=136, V=5000, ignore_frac=0.1),
             custom("noalloc_b", N=520, H=264, V=6208, ignore_frac=0.05)]
    for w in cases:
        assert flce.workspace_size(w.N, w.H, w.V) <= flce.NOALLOC_SCRATCH_BYTES
    for w in cases:  # two calls in a row, different sizes, one shared scratch array
        X, W, y = (t.cuda() for t in make_inputs(w))
        ref_loss, ref_dX, ref_dW = F.forward_backward(X, W, y)
        loss, dX, dW = flce.forward_backward_noalloc(X, W, y)
        assert_loss_close(loss, ref_loss, f"{w.name} loss")
        assert_grad_close(_np(dX), _np(ref_dX), f"{w.name} dX")
        assert_grad_close(_np(dW), _np(ref_dW), f"{w.name} dW")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Rejected on the host from the sizes alone, before any device work."""
    from lm_head_linear_03_b200 import flce
    import __graft_entry__
    __graft_entry__.build()
    lib = flce.load_library()
    fake = ctypes.c_void_p(1 << 20)
    loss = ctypes.c_float(0.0)
    N, H, V = 8192, 4096, 128256
    assert flce.workspace_size(N, H, V) > flce.NOALLOC_SCRATCH_BYTES
    st = lib.flce_forward_backward_noalloc(fake, fake, fake, N, H, V, -100, ctypes.byref(loss), fake, fake, None)
    assert st == 3  # FLCE_ERR_WORKSPACE_TOO_SMALL


@pytest.mark.gpu
def test_noalloc_reorders_rows_when_its_scratch_has_room():
    """The fixed scratch holds the packed-X area for small problems, so scattered
    ignored rows are reordered there too; results against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_head_linear_03_b200 import flce
    from oracle import flce_oracle as O
    w = custom("noalloc_reorder", N=1100, H=256, V=5000, ignore_frac=0.5)
    assert flce.workspace_size_reorder(w.N, w.H) <= flce.NOALLOC_SCRATCH_BYTES
    X, W, y = make_inputs(w)
    loss, dX, dW = flce.forward_backward_noalloc(X.cuda(), W.cuda(), y.cuda())
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(loss, rl)
    assert_grad_close(dX.float().cpu().numpy().astype("float64"), rdX, "dX")
    assert_grad_close(dW.float().cpu().numpy().astype("float64"), rdW, "dW")
    assert torch.count_nonzero(dX[(y == -100).cuda()]).item() == 0


@pytest.mark.gpu
def test_noalloc_keeps_the_order_when_only_the_base_size_fits():
    """A problem whose flce_workspace_size fits the fixed scratch but whose
    reorder workspace does not is accepted; the call keeps the caller's row
    order and still matches the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_head_linear_03_b200 import flce
    from oracle import flce_oracle as O
    w = custom("noalloc_base_only", N=1000, H=4096, V=3000, ignore_frac=0.5)
    assert flce.workspace_size(w.N, w.H, w.V) <= flce.NOALLOC_SCRATCH_BYTES < flce.workspace_size_reorder(w.N, w.H)
    X, W, y = make_inputs(w)
    loss, dX, dW = flce.forward_backward_noalloc(X.cuda(), W.cuda(), y.cuda())
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(loss, rl)
    assert_grad_close(dX.float().cpu().numpy().astype("float64"), rdX, "dX")
    assert_grad_close(dW.float().cpu().numpy().astype("float64"), rdW, "dW")
