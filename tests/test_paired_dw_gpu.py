"""dW items that pair two hidden tiles (256 x 512 in both accumulator buffers).

Pass 2 pairs the hidden tiles of its dW items when a chunk holds more than
three rounds of G tiles for the 74 SM pairs (more than 222 token x vocabulary
tiles), the regime of the large workloads.  These shapes enter that regime at
sizes the fp64 oracle finishes in seconds, and cover what the pairing meets:
an even and an odd number of hidden tiles (the last one alone), a ragged last
hidden tile inside a pair, scattered ignored rows (reordered rows), and a
prompt mask whose all-ignored token tiles the paired contraction skips at its
start, where a paired item runs its first half alone.  Every element is
compared with the oracle, through the plain entry and through the
asynchronous entry on a workspace that lets the call reorder rows.
"""
import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs
from test_parity_full_gpu import check_against_full_oracle

pytestmark = pytest.mark.gpu

PAIRED = [
    custom("paired_even_h", N=7424, H=1024, V=4100, ignore_frac=0.05),        # 29 x 8 tiles, 4 hidden tiles
    custom("paired_odd_h", N=7300, H=1200, V=2300, ignore_frac=0.3),          # 5 hidden tiles, the last ragged
    custom("paired_ragged_pair", N=7700, H=1288, V=6200, ignore_frac=0.1),    # 6 tiles, the 6th holds 8 columns
    custom("paired_prompt_mask", N=8192, H=776, V=2100, ignore_prefix=2600),  # 10 whole tiles ignored up front
]


def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    F.load_library()
    return F


@pytest.mark.parametrize("w", PAIRED, ids=lambda w: w.name)
@pytest.mark.parametrize("entry", ["plain", "async_reorder"])
def test_paired_dw_items_against_oracle(w, entry):
    F = _lib()
    X, W, y = make_inputs(w)
    if entry == "plain":
        loss, dX, dW = F.forward_backward(X.cuda(), W.cuda(), y.cuda())
    else:
        ws = F.alloc_workspace(w.N, w.H, w.V, reorder=True)
        loss_t, status, dX, dW = F.forward_backward_async(X.cuda(), W.cuda(), y.cuda(), workspace=ws)
        torch.cuda.synchronize()
        assert status.item() == 0
        loss = loss_t.item()
    check_against_full_oracle(X, W, y, loss, dX.cpu(), dW.cpu(), w.name, n_expected=w.N - w.n_ignored)


def test_paired_dw_items_repeat_bit_identically():
    """A fixed order of k-blocks in both halves: two calls give the same bits."""
    F = _lib()
    X, W, y = make_inputs(PAIRED[1])
    X, W, y = X.cuda(), W.cuda(), y.cuda()
    _, dX1, dW1 = F.forward_backward(X, W, y)
    _, dX2, dW2 = F.forward_backward(X, W, y)
    assert torch.equal(dX1, dX2) and torch.equal(dW1, dW2)


@pytest.mark.parametrize("w", PAIRED[1:3], ids=lambda w: w.name)
def test_paired_dw_items_through_the_host_entry(w):
    """The host-buffer entry: W in pieces (pass 1 per piece), pass 2 in
    sections with dW copied back per section, on shapes that pair dW items."""
    F = _lib()
    X, W, y = make_inputs(w)
    hX, hW, hy = X.pin_memory(), W.pin_memory(), y.pin_memory()
    dev = (torch.empty_like(X, device="cuda"), torch.empty_like(W, device="cuda"),
           torch.empty_like(y, device="cuda"), torch.empty_like(X, device="cuda"),
           torch.empty_like(W, device="cuda"), F.alloc_workspace(w.N, w.H, w.V))
    loss, hdX, hdW = F.forward_backward_host(hX, hW, hy, dev)
    check_against_full_oracle(X, W, y, loss, hdX, hdW, w.name + " host", n_expected=w.N - w.n_ignored)


@pytest.mark.parametrize("sections", [1, 3, 8])
def test_paired_dw_items_in_sections_match_one_launch(sections):
    """Pass 2 split into launches over whole chunks runs the same items in
    the same order: bit-identical to the single launch."""
    F = _lib()
    w = PAIRED[2]
    X, W, y = (t.cuda() for t in make_inputs(w))
    ws = F.alloc_workspace(w.N, w.H, w.V)
    l1, s1, dX1, dW1 = F.forward_backward_async(X, W, y, workspace=ws)
    torch.cuda.synchronize()
    dX1, dW1, l1 = dX1.clone(), dW1.clone(), l1.item()
    l2, s2, dX2, dW2, events, rows = F.forward_backward_sections(X, W, y, sections=sections, workspace=ws)
    torch.cuda.synchronize()
    assert s1.item() == 0 and s2.item() == 0
    assert rows[0] == 0 and rows[-1] == w.V
    assert l2.item() == l1 and torch.equal(dX2, dX1) and torch.equal(dW2, dW1)
