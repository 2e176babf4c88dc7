"""CUDA path against the fp64 oracle, element by element, through the C ABI.

Tolerances are the ones the target states: loss relative error <= 1e-4; dX and
dW relative Frobenius error <= 1e-2 and max-abs error <= 2^-7 * max|grad|.
"""
import math

import numpy as np
import pytest
import torch

from lm_head_linear_03_b200.inputs import WORKLOADS, custom, make_inputs
from oracle import flce_oracle as O

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-4
FRO_RTOL = 1e-2
MAXABS_FRAC = 2.0 ** -7


def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    F.load_library()
    return F


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def assert_grad_close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    nref = np.linalg.norm(ref)
    if nref == 0.0:
        assert np.all(got == 0.0), f"{what}: expected exact zeros"
        return
    fro = np.linalg.norm(got - ref) / nref
    mx = np.max(np.abs(got - ref))
    lim = MAXABS_FRAC * np.max(np.abs(ref))
    assert fro <= FRO_RTOL, f"{what}: relative Frobenius error {fro:.3e}"
    assert mx <= lim, f"{what}: max-abs error {mx:.3e} > {lim:.3e}"


def assert_loss_close(got, ref, what="loss"):
    if ref == 0.0:
        assert got == 0.0, f"{what}: {got} != 0"
        return
    assert abs(got - ref) <= LOSS_RTOL * abs(ref), f"{what}: {got} vs {ref}"


def run_full_oracle_case(X, W, y, ignore_index=-100):
    F = _lib()
    loss, dX, dW = F.forward_backward(X.cuda(), W.cuda(), y.cuda(), ignore_index)
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y, ignore_index)
    assert_loss_close(loss, rl)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")
    return loss, dX, dW


# Sizes the oracle finishes in seconds that still span several 128 x 256 tiles,
# several 2048-wide vocabulary chunks and ragged tails in N, H and V.
SMALL = [
    WORKLOADS["tiny"],
    custom("ragged_all_dims", N=300, H=136, V=5000, ignore_frac=0.1),
    custom("multi_chunk_tail64", N=520, H=264, V=6208, ignore_frac=0.05),   # V mod 256 = 64
    custom("single_token", N=1, H=64, V=300),
    custom("h_min", N=130, H=8, V=700, ignore_frac=0.2),
    custom("tiny_vocab", N=200, H=128, V=2, ignore_frac=0.1),
    custom("vocab_below_tile", N=129, H=96, V=100),
    custom("all_valid_zipf", N=384, H=512, V=9000, targets="zipf"),
    custom("prompt_mask", N=640, H=256, V=3000, ignore_prefix=200),
    custom("long_k", N=256, H=4096, V=1024, ignore_frac=0.1),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_against_full_oracle(w):
    X, W, y = make_inputs(w)
    run_full_oracle_case(X, W, y)


@pytest.mark.parametrize("N,H,V,frac", [(70000, 64, 600, 0.3), (70000, 32, 300, 0.0), (8, 64, 300000, 0.25)])
def test_many_tiles_or_wide_vocab(N, H, V, frac):
    """More than 256 token tiles (the row-order kernel's loops over tiles take
    several passes), and a vocabulary of 300000 with a handful of rows."""
    w = custom(f"extent_{N}_{H}_{V}", N=N, H=H, V=V, ignore_frac=frac)
    X, W, y = make_inputs(w)
    run_full_oracle_case(X, W, y)


def test_all_rows_ignored_gives_zero():
    w = custom("all_ignored", N=200, H=64, V=1000)
    X, W, y = make_inputs(w)
    y[:] = -100
    loss, dX, dW = run_full_oracle_case(X, W, y)
    assert loss == 0.0
    assert torch.count_nonzero(dX).item() == 0 and torch.count_nonzero(dW).item() == 0


def test_zero_weight_gives_log_v():
    w = custom("w_zero", N=257, H=64, V=5000, ignore_frac=0.1)
    X, W, y = make_inputs(w)
    W.zero_()
    loss, dX, _ = run_full_oracle_case(X, W, y)
    assert abs(loss - math.log(5000)) <= 1e-6 * math.log(5000)
    assert torch.count_nonzero(dX).item() == 0


def test_large_logit_range():
    """|z| up to ~80: the online max shift must keep every exponential finite."""
    w = custom("large_logits", N=256, H=256, V=3000, ignore_frac=0.1, x_std=4.0, w_std=0.3)
    X, W, y = make_inputs(w)
    z = X.float() @ W.float().T
    assert z.abs().max().item() > 60
    run_full_oracle_case(X, W, y)


def test_target_zero_everywhere():
    w = custom("all_target_zero", N=300, H=128, V=2500)
    X, W, y = make_inputs(w)
    y[:] = 0
    run_full_oracle_case(X, W, y)


def test_other_ignore_index():
    w = custom("ignore_minus_one", N=256, H=128, V=1500)
    X, W, y = make_inputs(w)
    y[::7] = -1
    run_full_oracle_case(X, W, y, ignore_index=-1)


def test_repeat_calls_identical():
    """Same inputs, same workspace: bit-identical results (no atomics in the sums)."""
    F = _lib()
    X, W, y = (t.cuda() for t in make_inputs(custom("det", N=384, H=256, V=4500, ignore_frac=0.1)))
    ws = F.alloc_workspace(384, 256, 4500)
    l1, dX1, dW1 = F.forward_backward(X, W, y, workspace=ws)
    l2, dX2, dW2 = F.forward_backward(X, W, y, workspace=ws)
    assert l1 == l2 and torch.equal(dX1, dX2) and torch.equal(dW1, dW2)


def test_async_matches_sync():
    F = _lib()
    X, W, y = (t.cuda() for t in make_inputs(WORKLOADS["tiny"]))
    l1, dX1, dW1 = F.forward_backward(X, W, y)
    loss, status, dX2, dW2 = F.forward_backward_async(X, W, y)
    torch.cuda.synchronize()
    assert status.item() == 0 and loss.item() == l1
    assert torch.equal(dX1, dX2) and torch.equal(dW1, dW2)


@pytest.mark.parametrize("N,H,V", [(300, 136, 5000), (700, 256, 9000), (256, 128, 700)])
def test_host_entry_matches_device_entry(N, H, V):
    """The host-buffer entry copies W in pieces and runs pass 1 per piece (its
    log-sum-exp partials merge in another order) and pass 2 in sections with
    dW copied back per section: the oracle's tolerances hold for both entries,
    and they agree with each other to rounding."""
    F = _lib()
    w = custom(f"host_{N}_{H}_{V}", N=N, H=H, V=V, ignore_frac=0.1)
    X, W, y = make_inputs(w)
    l1, dX1, dW1 = F.forward_backward(X.cuda(), W.cuda(), y.cuda())
    hX, hW, hy = X.pin_memory(), W.pin_memory(), y.pin_memory()
    dev = (torch.empty_like(X, device="cuda"), torch.empty_like(W, device="cuda"),
           torch.empty_like(y, device="cuda"), torch.empty_like(X, device="cuda"),
           torch.empty_like(W, device="cuda"), F.alloc_workspace(w.N, w.H, w.V))
    l2, hdX, hdW = F.forward_backward_host(hX, hW, hy, dev)
    rl, rdX, rdW, _, _ = O.flce_reference(X, W, y)
    assert_loss_close(l2, rl)
    assert_grad_close(_np(hdX), rdX, "host dX")
    assert_grad_close(_np(hdW), rdW, "host dW")
    assert abs(l1 - l2) <= 1e-6 * abs(l1)
    for a, b in ((dX1.cpu(), hdX), (dW1.cpu(), hdW)):
        d = (a.float() - b.float()).abs().max().item()
        assert d <= 2.0 ** -8 * a.float().abs().max().item(), d


def test_target_out_of_range_reported():
    F = _lib()
    X, W, y = make_inputs(custom("oor", N=256, H=64, V=1000))
    y[17] = 1000
    with pytest.raises(F.FlceError) as e:
        F.forward_backward(X.cuda(), W.cuda(), y.cuda())
    assert e.value.status == 4
    y[17] = -5
    with pytest.raises(F.FlceError) as e:
        F.forward_backward(X.cuda(), W.cuda(), y.cuda())
    assert e.value.status == 4
    # the device stays usable
    y[17] = 3
    run_full_oracle_case(X, W, y)


def test_host_argument_errors():
    F = _lib()
    X = torch.zeros(64, 12, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(100, 12, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(64, dtype=torch.int32, device="cuda")
    with pytest.raises(F.FlceError) as e:  # H % 8 != 0
        F.forward_backward(X, W, y)
    assert e.value.status == 2
    X = torch.zeros(64, 16, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(100, 16, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(F.FlceError) as e:
        F.forward_backward_async(X, W, y, workspace=small)
    assert e.value.status == 3


def test_workspace_within_budget():
    F = _lib()
    assert F.workspace_size(8192, 4096, 128256) == F.workspace_size(8192, 4096, 1)
    assert F.workspace_size(8192, 4096, 128256) <= 0.05 * 8192 * 128256 * 2
    assert F.workspace_size(4096, 2304, 256000) <= 0.05 * 4096 * 256000 * 2


def test_peak_device_bytes_equal_buffers_plus_workspace():
    """No hidden allocation: the call's peak is inputs + outputs + workspace."""
    F = _lib()
    w = custom("peak", N=1024, H=512, V=20000, ignore_frac=0.1)
    X, W, y = (t.cuda() for t in make_inputs(w))
    dX, dW = torch.empty_like(X), torch.empty_like(W)
    ws = F.alloc_workspace(w.N, w.H, w.V)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    F.forward_backward(X, W, y, dX=dX, dW=dW, workspace=ws)
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == base


def _ex_case(w, **kw):
    F = _lib()
    X, W, y = make_inputs(w)
    loss, status, rl, dX, dW = F.forward_backward_ex(X.cuda(), W.cuda(), y.cuda(), **kw)
    torch.cuda.synchronize()
    assert status.item() == 0
    return X, W, y, loss.item(), rl, dX, dW


def test_reduction_sum():
    w = custom("red_sum", N=300, H=136, V=5000, ignore_frac=0.1)
    X, W, y, loss, rl, dX, dW = _ex_case(w, reduction="sum", row_loss=True)
    ref, rdX, rdW, _, _, rows = O.flce_reference(X, W, y, reduction="sum", return_rows=True)
    assert_loss_close(loss, ref)
    assert_grad_close(_np(dX), rdX, "dX sum")
    assert_grad_close(_np(dW), rdW, "dW sum")
    r = rl.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(r - rows)) <= LOSS_RTOL * np.max(np.abs(rows))


def test_reduction_none_with_upstream_weights():
    """Per-row upstream gradients of both signs, the fused-linear core a
    preference loss builds on (weighted per-token log-probabilities)."""
    w = custom("red_none", N=520, H=264, V=6208, ignore_frac=0.05)
    g = torch.randn(520, generator=torch.Generator().manual_seed(5)).float()
    X, W, y, loss, rl, dX, dW = _ex_case(w, reduction="none", grad_row_scale=g.cuda(), row_loss=True)
    ref, rdX, rdW, _, _, rows = O.flce_reference(X, W, y, reduction="none", grad_row_scale=g.double().numpy(),
                                                 return_rows=True)
    assert abs(loss - ref) <= LOSS_RTOL * float(np.sum(np.abs(g.double().numpy() * rows)))
    assert_grad_close(_np(dX), rdX, "dX none")
    assert_grad_close(_np(dW), rdW, "dW none")
    r = rl.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(r - rows)) <= LOSS_RTOL * np.max(np.abs(rows))
    assert np.all(r[y.numpy() == -100] == 0.0)


def test_forward_only_matches_full_call():
    F = _lib()
    w = custom("fwd_only", N=384, H=256, V=4500, ignore_frac=0.1)
    X, W, y = (t.cuda() for t in make_inputs(w))
    full, _, _ = F.forward_backward(X, W, y)
    loss, status, rl, dX, dW = F.forward_backward_ex(X, W, y, grads=False, row_loss=True)
    torch.cuda.synchronize()
    assert status.item() == 0 and dX is None and dW is None
    assert loss.item() == full
    ref, _, _, _, _, rows = O.flce_reference(X, W, y, return_rows=True)
    r = rl.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(r - rows)) <= LOSS_RTOL * np.max(np.abs(rows))


@pytest.mark.parametrize("N,H,V,ignored", [
    (1100, 136, 5000, slice(0, 600)),      # prompt mask covering two whole 256-row tiles
    (1024, 264, 6208, slice(256, 512)),    # one whole tile in the middle
    (768, 64, 2500, slice(0, 768)),        # every tile (all rows ignored)
])
def test_whole_ignored_token_tiles_are_skipped(N, H, V, ignored):
    """Tiles whose rows are all ignored skip pass 1, the G and dX tiles and their
    k-blocks of dW; results stay equal to the oracle's."""
    w = custom(f"skip_{N}_{H}_{V}", N=N, H=H, V=V, ignore_frac=0.05)
    X, W, y = make_inputs(w)
    y[ignored] = -100
    loss, dX, dW = run_full_oracle_case(X, W, y)
    assert torch.count_nonzero(dX[ignored]).item() == 0


def test_bounded_waits_give_up_and_report_timeout():
    """Failure detection without a fault: waits on an event that never comes
    end after their limit with FLCE_ERR_TIMEOUT, and the device stays usable."""
    F = _lib()
    from lm_head_linear_03_b200 import flce
    import time
    t0 = time.perf_counter()
    st = flce.probe_bounded_wait(2_000_000)  # 2 ms per wait
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert st.tolist() == [5, 5, 0]
    run_full_oracle_case(*make_inputs(WORKLOADS["tiny"]))


@pytest.mark.parametrize("shape", [(700, 256, 5000), (7424, 1024, 4100)], ids=["single_dw", "paired_dw"])
def test_pass2_starved_waits_give_up_and_report_timeout(shape):
    """The GEMM kernels' own waits: a call whose dW items wait for one more
    G tile than the queue produces ends with FLCE_ERR_TIMEOUT within seconds
    (each SM pair winds down, both CTAs together), and the next call on the
    device matches the oracle.  The second shape runs its dW items as paired
    256 x 512 tiles (a chunk holds more than three rounds of G tiles)."""
    _lib()
    from lm_head_linear_03_b200 import flce
    import time
    N, H, V = shape
    w = custom(f"starved_dw_{N}", N=N, H=H, V=V, ignore_frac=0.1)
    X, W, y = make_inputs(w)
    Xd, Wd, yd = X.cuda(), W.cuda(), y.cuda()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    st = flce.probe_pass2_timeout(Xd, Wd, yd, timeout_ns=5_000_000)  # 5 ms per wait
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 10.0
    assert st.item() == 5
    run_full_oracle_case(X, W, y)


def test_mean_over_external_count():
    """The data-parallel hook: the mean divides by a count from outside the call
    (all ranks' valid targets); equals the oracle with weights 1/count."""
    F = _lib()
    w = custom("mean_count", N=300, H=136, V=5000, ignore_frac=0.1)
    X, W, y = make_inputs(w)
    count = 1000
    loss, status, _, dX, dW = F.forward_backward_ex(X.cuda(), W.cuda(), y.cuda(),
                                                    mean_count=torch.tensor([count], dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert status.item() == 0
    valid = (y != -100).numpy()
    ref, rdX, rdW, _, _ = O.flce_reference(X, W, y, reduction="none", grad_row_scale=np.where(valid, 1.0 / count, 0.0))
    assert_loss_close(loss.item(), ref)
    assert_grad_close(_np(dX), rdX, "dX")
    assert_grad_close(_np(dW), rdW, "dW")
