"""Data-parallel host logic on CPU with gloo (world size 2).

Each rank holds a different token shard; the per-rank compute is the fp64 oracle
taking the mean over the count all ranks share.  After the exchanges the
loss and dW must be the whole batch's and each rank's dX its rows of the batch
dX: the oracle on the concatenated batch decides.
"""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch(seed=0, N=40, H=12, V=50):
    r = np.random.default_rng(seed)
    X = r.standard_normal((N, H))
    W = r.standard_normal((V, H)) * 0.3
    y = r.integers(0, V, size=N)
    y[r.permutation(N)[:7]] = -100
    y[:5] = -100  # rank 0 gets more ignored rows than rank 1
    return X, W, y


def _oracle_call(X, W, y, ignore_index, mean_count):
    from oracle import flce_oracle as O
    n = int(mean_count.item())
    valid = (y != ignore_index).numpy()
    loss, dX, dW, _, _ = O.flce_reference(X.numpy(), W.numpy(), y.numpy(), ignore_index, reduction="none",
                                          grad_row_scale=np.where(valid, 1.0 / n, 0.0))
    return (torch.tensor([loss], dtype=torch.float64), torch.zeros(1, dtype=torch.int32), torch.tensor(dX),
            torch.tensor(dW))


def _oracle_count(y, ignore_index):
    from oracle import flce_oracle as O
    return torch.tensor([int(O.valid_mask(y.numpy(), 1 << 30, ignore_index).sum())], dtype=torch.int32)


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from lm_head_linear_03_b200.parallel import dp_forward_backward
    dist.init_process_group("gloo", rank=rank, world_size=world)
    X, W, y = _batch()
    shard = slice(rank * 20, (rank + 1) * 20)
    loss, dX, dW = dp_forward_backward(torch.tensor(X[shard]), torch.tensor(W), torch.tensor(y[shard]),
                                       local_call=_oracle_call, count_call=_oracle_count)
    q.put((rank, float(loss.item()), dX.numpy(), dW.numpy()))
    dist.destroy_process_group()


def test_data_parallel_matches_whole_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, loss, dX, dW = q.get(timeout=120)
        res[r] = (loss, dX, dW)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    from oracle import flce_oracle as O
    X, W, y = _batch()
    loss, dX, dW, _, _ = O.flce_reference(X, W, y)
    for r in range(2):
        assert abs(res[r][0] - loss) <= 1e-12 * abs(loss)
        np.testing.assert_allclose(res[r][1], dX[r * 20:(r + 1) * 20], rtol=1e-10, atol=1e-15)
        np.testing.assert_allclose(res[r][2], dW, rtol=1e-10, atol=1e-15)
