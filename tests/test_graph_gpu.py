"""The asynchronous entry captured in a CUDA graph.

A call enqueues only stream work fixed by its pointers and sizes: memsets and
kernel launches whose tensor maps travel by value.  Every decision that
depends on the data is taken on the device: which token tiles are skipped,
whether the rows are reordered, and the mean's count.  So one captured call,
replayed, computes the head on whatever the buffers hold at replay time.
Each replay is checked against a direct call on the same inputs
(bit-identical) and against the fp64 oracle."""
import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs
from oracle import flce_oracle as O
from test_parity_gpu import _lib, _np, assert_grad_close, assert_loss_close

pytestmark = pytest.mark.gpu

# 5 token tiles (the last one ragged), 3 vocabulary chunks (the last one ragged)
N, H, V = 1100, 192, 4700

# in replay order: rows kept in place, then reordered (scattered ignores),
# then two whole tiles skipped in place (prompt mask), then both
CASES = [
    dict(ignore_frac=0.0),
    dict(ignore_frac=0.6),
    dict(ignore_prefix=512),
    dict(ignore_frac=0.3, ignore_prefix=300),
]
EXPECT_REORDERED = [False, True, False, True]


def _reorder_rule(y):
    """Rows are reordered when the valid rows, packed, fill fewer 256-row
    tiles than the tiles that hold a valid row now."""
    v = (y != -100).numpy().astype(np.int64)
    nonempty = int((np.add.reduceat(v, np.arange(0, len(v), 256)) > 0).sum())
    return -(-int(v.sum()) // 256) < nonempty


def _buffers():
    dev = "cuda"
    return (torch.empty(1, dtype=torch.float32, device=dev), torch.empty(1, dtype=torch.int32, device=dev),
            torch.empty(N, H, dtype=torch.bfloat16, device=dev), torch.empty(V, H, dtype=torch.bfloat16, device=dev))


def test_captured_call_replays_on_new_inputs():
    F = _lib()
    inputs = [make_inputs(custom(f"graph{k}", N=N, H=H, V=V, seed=k, **kw)) for k, kw in enumerate(CASES)]
    Xd = torch.empty(N, H, dtype=torch.bfloat16, device="cuda")
    Wd = torch.empty(V, H, dtype=torch.bfloat16, device="cuda")
    yd = torch.empty(N, dtype=torch.int32, device="cuda")
    ws = F.alloc_workspace(N, H, V, reorder=True)
    out = _buffers()

    def load(k):
        X, W, y = inputs[k]
        Xd.copy_(X)
        Wd.copy_(W)
        yd.copy_(y)

    # a direct call first: it sets up the library (kernel attributes, tensor-map encoder)
    load(0)
    F.forward_backward_async(Xd, Wd, yd, out=out, workspace=ws)
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.graph(graph, stream=side):
        F.forward_backward_async(Xd, Wd, yd, out=out, workspace=ws)

    direct = _buffers()
    for k in range(len(CASES)):
        load(k)
        for t in out:
            t.fill_(-1)
        graph.replay()
        torch.cuda.synchronize()
        assert out[1].item() == 0, (k, out[1].item())
        reordered, n_valid = F.row_order_info(ws)

        F.forward_backward_async(Xd, Wd, yd, out=direct, workspace=ws)
        torch.cuda.synchronize()
        for a, b, what in zip(out, direct, ("loss", "status", "dX", "dW")):
            assert torch.equal(a, b), f"case {k}: replayed {what} differs from the direct call"

        X, W, y = inputs[k]
        ref, rdX, rdW, _, n = O.flce_reference(X, W, y)
        assert n_valid == n
        assert reordered == _reorder_rule(y) == EXPECT_REORDERED[k], (k, reordered)
        assert_loss_close(out[0].item(), ref, f"loss case {k}")
        assert_grad_close(_np(out[2]), rdX, f"dX case {k}")
        assert_grad_close(_np(out[3]), rdW, f"dW case {k}")
        assert torch.count_nonzero(out[2][(y == -100).cuda()]).item() == 0
    del graph


def test_replays_back_to_back_without_host_sync():
    """Several replays queued on one stream: each starts from a clean
    workspace (the captured memsets), so the last result equals one call."""
    F = _lib()
    X, W, y = (t.cuda() for t in make_inputs(custom("graph_b2b", N=N, H=H, V=V, ignore_frac=0.25)))
    ws = F.alloc_workspace(N, H, V)
    out = _buffers()
    F.forward_backward_async(X, W, y, out=out, workspace=ws)
    torch.cuda.synchronize()
    once = tuple(t.clone() for t in out)

    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.graph(graph, stream=side):
        F.forward_backward_async(X, W, y, out=out, workspace=ws)
    for _ in range(5):
        graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(out, once):
        assert torch.equal(a, b)
    del graph
