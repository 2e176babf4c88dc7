"""The multi-device glue with its default CUDA calls and NCCL, on the one GPU a
test run has: a process group of one rank (NCCL), through which the data- and
vocabulary-parallel heads run end to end (count, exchanges, the library's
calls) and must match the fp64 oracle.  With one rank every collective is the
identity, so the exchanges' arithmetic is covered by the gloo tests on CPU;
here the device path runs.  Also: the sectioned call behind the overlapped dW
all-reduce is bit-identical to the unsplit call."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs
from oracle import flce_oracle as O
from test_parity_gpu import assert_grad_close, assert_loss_close

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield dist
    dist.destroy_process_group()


def _case():
    w = custom("parallel_gpu", N=700, H=264, V=9000, ignore_frac=0.15)
    X, W, y = make_inputs(w)
    return X, W, y


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def test_data_parallel_head_single_rank(nccl_group):
    from lm_head_linear_03_b200.parallel import dp_forward_backward
    X, W, y = _case()
    loss, dX, dW = dp_forward_backward(X.cuda(), W.cuda(), y.cuda())
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(loss.item(), rl)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")


@pytest.mark.parametrize("sections", [1, 3, 8])
def test_overlapped_data_parallel_head_single_rank(nccl_group, sections):
    import lm_head_linear_03_b200 as F
    from lm_head_linear_03_b200.parallel import dp_forward_backward_overlapped
    X, W, y = (t.cuda() for t in _case())
    loss, dX, dW = dp_forward_backward_overlapped(X, W, y, sections=sections)
    rl, rdX, rdW, _, _ = O.flce_reference(X.cpu(), W.cpu(), y.cpu())
    assert_loss_close(loss.item(), rl)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")
    # the sectioned call alone: same sums in the same order as the unsplit call
    l1, s1, dX1, dW1 = F.forward_backward_async(X, W, y)
    l2, s2, dX2, dW2, events, rows = F.forward_backward_sections(X, W, y, sections=sections)
    torch.cuda.synchronize()
    assert s1.item() == 0 and s2.item() == 0
    assert l1.item() == l2.item() and torch.equal(dX1, dX2) and torch.equal(dW1, dW2)
    assert rows[0] == 0 and rows[-1] == W.shape[0] and all(a <= b for a, b in zip(rows, rows[1:]))
    assert all(e.query() for e in events)


def test_vocab_parallel_head_single_rank(nccl_group):
    from lm_head_linear_03_b200.parallel import vp_forward_backward
    X, W, y = _case()
    loss, dX, dW = vp_forward_backward(X.cuda(), W.cuda(), y.cuda(), 0, W.shape[0])
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(loss.item(), rl)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")


def test_count_valid_matches_the_targets():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    for N, frac in ((1, 0.0), (700, 0.15), (70000, 0.5), (300, 1.0)):
        y = make_inputs(custom("count", N=N, H=8, V=50, ignore_frac=frac))[2]
        n = F.count_valid(y.cuda())
        assert n.item() == int((y != -100).sum()), (N, frac)
