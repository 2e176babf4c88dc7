"""Vocabulary-parallel head through the C ABI, its shards run one after
another on one GPU (no kernel waits on another shard): step 1 on every shard,
the all-gather as a stack, step 3 on every shard, the dX all-reduce as a sum.
Each step is checked against the fp64 oracle: the shard statistics against
its shard_stats, the loss, summed dX and concatenated dW against the whole-
vocabulary head."""
import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs
from oracle import flce_oracle as O
from test_parity_gpu import _lib, _np, assert_grad_close, assert_loss_close

pytestmark = pytest.mark.gpu


def _run_shards(X, W, y, bounds, mean_count=None):
    F = _lib()
    Xd, yd = X.cuda(), y.cuda()
    V = W.shape[0]
    shards = [(v0, v1, W[v0:v1].contiguous().cuda()) for v0, v1 in zip(bounds[:-1], bounds[1:])]
    lses, zys = [], []
    for v0, v1, Ws in shards:
        lse, zy, st = F.vp_shard_stats(Xd, Ws, yd, v0, V)
        torch.cuda.synchronize()
        assert st.item() == 0
        ref_lse, ref_zy = O.shard_stats(X, W[v0:v1], y, v0)
        valid = (y != -100).numpy()
        got_lse = lse.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(got_lse - ref_lse)[valid]) <= 1e-4 * max(1.0, np.max(np.abs(ref_lse))), (v0, v1)
        got_zy = zy.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(got_zy - ref_zy)) <= 1e-4 * max(1.0, np.max(np.abs(ref_zy))), (v0, v1)
        assert np.all(got_zy[ref_zy == 0.0] == 0.0)  # rows whose target is elsewhere, or ignored
        lses.append(lse)
        zys.append(zy)
    all_lse = torch.stack(lses).contiguous()
    all_zy = torch.stack(zys).contiguous()
    losses, dWs = [], []
    dX = torch.zeros(X.shape, dtype=torch.float32, device="cuda")
    for v0, v1, Ws in shards:
        loss, st, dXp, dWs_ = F.vp_backward(Xd, Ws, yd, v0, V, all_lse, all_zy, mean_count=mean_count)
        torch.cuda.synchronize()
        assert st.item() == 0
        losses.append(loss.item())
        dX += dXp.float()
        dWs.append(dWs_)
    return losses, dX, torch.cat(dWs)


CASES = [
    # (workload, shard bounds)
    (custom("vp_three_uneven", N=600, H=256, V=9000, ignore_frac=0.1), [0, 2500, 2503, 9000]),
    (custom("vp_ragged", N=333, H=136, V=5000, ignore_frac=0.2), [0, 700, 4100, 5000]),
    (custom("vp_long_k", N=256, H=4096, V=3000, ignore_frac=0.05), [0, 1500, 3000]),
    (custom("vp_single_shard", N=300, H=128, V=4000, ignore_frac=0.1), [0, 4000]),
    (custom("vp_eight", N=512, H=192, V=6000, targets="zipf"), [0, 750, 1500, 2250, 3000, 3750, 4500, 5250, 6000]),
]


@pytest.mark.parametrize("w,bounds", CASES, ids=[c[0].name for c in CASES])
def test_vocab_shards_match_whole_vocabulary(w, bounds):
    X, W, y = make_inputs(w)
    losses, dX, dW = _run_shards(X, W, y, bounds)
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    for loss in losses:
        assert_loss_close(loss, rl)
    assert max(losses) == min(losses)  # every shard merges the same statistics in the same order
    assert_grad_close(dX.cpu().numpy().astype(np.float64), rdX, "dX (sum of shards)")
    assert_grad_close(_np(dW), rdW, "dW (shards concatenated)")


def test_shard_without_targets():
    w = custom("vp_no_targets", N=400, H=128, V=3000, ignore_frac=0.1)
    X, W, y = make_inputs(w)
    y[(y >= 1000) & (y < 2000)] = 5  # the middle shard holds no target
    losses, dX, dW = _run_shards(X, W, y, [0, 1000, 2000, 3000])
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(losses[0], rl)
    assert_grad_close(dX.cpu().numpy().astype(np.float64), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")


def test_shards_with_external_count():
    w = custom("vp_count", N=300, H=136, V=4000, ignore_frac=0.1)
    X, W, y = make_inputs(w)
    count = 900
    losses, dX, dW = _run_shards(X, W, y, [0, 1800, 4000],
                                 mean_count=torch.tensor([count], dtype=torch.int32).cuda())
    valid = (y != -100).numpy()
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y, reduction="none", grad_row_scale=np.where(valid, 1.0 / count, 0.0))
    assert_loss_close(losses[0], rl)
    assert_grad_close(dX.cpu().numpy().astype(np.float64), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")


def test_shard_target_out_of_whole_range_reported():
    F = _lib()
    w = custom("vp_bad_target", N=200, H=64, V=2000)
    X, W, y = make_inputs(w)
    y[17] = 2000  # outside the whole vocabulary, though inside no shard either
    _, _, st = F.vp_shard_stats(X.cuda(), W[:1000].contiguous().cuda(), y.cuda(), 0, 2000)
    torch.cuda.synchronize()
    assert st.item() == 4  # FLCE_ERR_TARGET_OUT_OF_RANGE
    y[17] = 1500  # another shard's target is fine for this one
    _, _, st = F.vp_shard_stats(X.cuda(), W[:1000].contiguous().cuda(), y.cuda(), 0, 2000)
    torch.cuda.synchronize()
    assert st.item() == 0
