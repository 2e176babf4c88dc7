"""Vocabulary-parallel host logic on CPU with gloo (world sizes 2 and 3).

Each rank holds a contiguous shard of W rows; X and y are replicated.  The
per-rank compute is fp64: the oracle's shard statistics for step 1, and for
step 3 a fake device call that forms the shard's G from the merged statistics.
After the all-gather and the dX all-reduce every rank must hold the whole
batch's loss and dX, and its dW rows must be the whole dW's: the oracle on the
unsharded vocabulary decides.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch(seed=3, N=30, H=10, V=47):
    r = np.random.default_rng(seed)
    X = r.standard_normal((N, H))
    W = r.standard_normal((V, H)) * 0.4
    y = r.integers(0, V, size=N)
    y[r.permutation(N)[:6]] = -100
    y[0] = V - 1
    return X, W, y


def _stats_call(X, W_shard, y, v0, V, ignore_index):
    from oracle import flce_oracle as O
    lse, zy = O.shard_stats(X.numpy(), W_shard.numpy(), y.numpy(), v0, ignore_index)
    return torch.tensor(lse), torch.tensor(zy), torch.zeros(1, dtype=torch.int32)


def _backward_call(X, W_shard, y, v0, V, all_lse, all_zy, ignore_index):
    """Fake device step 3: the merged statistics give lse and the loss; this
    shard's columns of G give its dW rows and its share of dX."""
    from oracle import flce_oracle as O
    lse, zy = O.merge_shard_stats(all_lse.numpy(), all_zy.numpy())
    Xn, Ws, yn = X.numpy(), W_shard.numpy(), y.numpy()
    valid = yn != ignore_index
    n = int(valid.sum())
    loss = float(np.where(valid, lse - zy, 0.0).sum() / n)
    G = np.exp(Xn @ Ws.T - lse[:, None])
    local = yn - v0
    inside = valid & (local >= 0) & (local < Ws.shape[0])
    G[np.nonzero(inside)[0], local[inside]] -= 1.0
    G *= np.where(valid, 1.0 / n, 0.0)[:, None]
    return (torch.tensor([loss], dtype=torch.float64), torch.zeros(1, dtype=torch.int32), torch.tensor(G @ Ws),
            torch.tensor(G.T @ Xn))


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from lm_head_linear_03_b200.parallel import vocab_shard_range, vp_forward_backward
    dist.init_process_group("gloo", rank=rank, world_size=world)
    X, W, y = _batch()
    V = W.shape[0]
    v0, v1 = vocab_shard_range(V, world, rank)
    loss, dX, dW = vp_forward_backward(torch.tensor(X), torch.tensor(W[v0:v1]), torch.tensor(y), v0, V,
                                       stats_call=_stats_call, backward_call=_backward_call)
    q.put((rank, v0, v1, float(loss.item()), dX.numpy(), dW.numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_vocab_parallel_matches_whole_vocabulary(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, v0, v1, loss, dX, dW = q.get(timeout=120)
        res[r] = (v0, v1, loss, dX, dW)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    from oracle import flce_oracle as O
    X, W, y = _batch()
    loss, dX, dW, _, _ = O.flce_reference(X, W, y)
    covered = []
    for r in range(world):
        v0, v1, l_r, dX_r, dW_r = res[r]
        covered.append((v0, v1))
        assert abs(l_r - loss) <= 1e-12 * abs(loss)
        np.testing.assert_allclose(dX_r, dX, rtol=1e-10, atol=1e-15)
        np.testing.assert_allclose(dW_r, dW[v0:v1], rtol=1e-10, atol=1e-15)
    assert sorted(covered)[0][0] == 0 and sorted(covered)[-1][1] == W.shape[0]
    assert all(a[1] == b[0] for a, b in zip(sorted(covered), sorted(covered)[1:]))


def test_vocab_shard_ranges_tile_the_vocabulary():
    sys.path.insert(0, ROOT)
    from lm_head_linear_03_b200.parallel import vocab_shard_range
    for V in (1, 7, 128256, 256000):
        for world in (1, 2, 3, 8):
            spans = [vocab_shard_range(V, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == V
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
