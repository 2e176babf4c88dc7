"""The host-buffer entry's timeline from the library's own record: every copy
and launch with its CUDA-event interval, in the order the entry overlaps them."""
import pytest
import torch

from lm_head_linear_03_b200.inputs import custom, make_inputs

pytestmark = pytest.mark.gpu
EPS = 1e-3  # ms: event timestamps resolve to about half a microsecond


def test_host_entry_timeline_follows_the_overlap():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lm_head_linear_03_b200 as F
    F.load_library()
    w = custom("timeline", N=1024, H=512, V=40000, ignore_frac=0.1)  # 157 vocabulary tiles, 20 chunks
    X, W, y = make_inputs(w)
    hX, hW, hy = X.pin_memory(), W.pin_memory(), y.pin_memory()
    dev = (torch.empty_like(X, device="cuda"), torch.empty_like(W, device="cuda"),
           torch.empty_like(y, device="cuda"), torch.empty_like(X, device="cuda"),
           torch.empty_like(W, device="cuda"), F.alloc_workspace(w.N, w.H, w.V))
    F.forward_backward_host(hX, hW, hy, dev)  # warm-up: copy stream and events made on first use
    F.profile_enable(True)
    try:
        F.forward_backward_host(hX, hW, hy, dev)
        tl = F.profile_timeline()
    finally:
        F.profile_enable(False)
    assert all(b <= e + EPS for _, b, e in tl)
    assert tl[0][0] == "copy_host_to_device" and abs(tl[0][1]) <= EPS  # X and y open the record
    h2d = [t for t in tl if t[0] == "copy_host_to_device"]
    d2h = [t for t in tl if t[0] == "copy_device_to_host"]
    p1 = [t for t in tl if t[0] == "pass1_logits_lse"]
    p2 = [t for t in tl if t[0] == "pass2_grad_dw_dx"]
    pieces, sections = 16, 16
    assert len(h2d) == 1 + pieces and len(p1) == pieces and len(p2) == sections
    assert len(d2h) == sections + 1
    # pass 1 on a W piece starts only once that piece has landed
    for (_, _, landed), (_, start, _) in zip(h2d[1:], p1):
        assert start >= landed - EPS
    # pass 2 after every pass-1 piece; each section's dW rows leave after the section
    assert p2[0][1] >= max(e for _, _, e in p1) - EPS
    for (_, _, done), (_, start, _) in zip(p2, d2h[:-1]):
        assert start >= done - EPS
    # dX and the loss last, after the last section
    assert d2h[-1][1] >= p2[-1][2] - EPS
    # the record is cleared by the read
    assert F.profile_timeline() == []
