"""The C ABI without a GPU: the library loads, exports every function the header
declares, and answers the host-only queries (no kernel is launched here)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(flce_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    from lm_head_linear_03_b200 import flce
    return flce.load_library()


def test_header_declares_entry_points():
    names = declared_functions()
    for must in ("flce_forward_backward", "flce_workspace_size", "flce_forward_backward_async"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_binding_covers_the_header():
    from lm_head_linear_03_b200 import flce
    assert set(declared_functions()) <= set(flce.EXPORTED)


def test_status_strings(lib):
    lib.flce_status_string.restype = ctypes.c_char_p
    assert lib.flce_status_string(0) == b"FLCE_OK"
    assert lib.flce_status_string(4) == b"FLCE_ERR_TARGET_OUT_OF_RANGE"
    assert lib.flce_status_string(99) == b"FLCE_UNKNOWN_STATUS"


def test_workspace_size_by_vocab(lib):
    from lm_head_linear_03_b200 import flce
    # the size depends on N and H only: the same for every vocabulary
    sizes = {flce.workspace_size(8192, 4096, v) for v in (1, 2, 4096, 32064, 128256, 256000, 1 << 24)}
    assert len(sizes) == 1, sizes
    base = sizes.pop()
    # the workspace that lets a call reorder token rows adds the N x H bf16 area
    assert flce.workspace_size_reorder(8192, 4096) == base + 8192 * 4096 * 2
    assert flce.workspace_size_reorder(4096, 2304) == flce.workspace_size(4096, 2304, 256000) + 4096 * 2304 * 2
    assert flce.workspace_size_reorder(300, 136) == flce.workspace_size(300, 136, 5) + (300 * 136 * 2 + 255) // 256 * 256
    # the Llama-3-8B head workload stays within 5% of its N x V x 2-byte logits
    assert flce.workspace_size(8192, 4096, 128256) <= 0.05 * 8192 * 128256 * 2
    # the benchmark's choice: the reorder workspace where it stays within that 5%
    assert not flce.reorder_fits(8192, 4096, 128256)
    assert flce.reorder_fits(4096, 2304, 256000)
    assert flce.workspace_size(0, 4096, 10) == 0
    assert flce.workspace_size(16, 12, 10) == 0  # H % 8 != 0
    assert flce.workspace_size_reorder(16, 12) == 0


def test_plan_is_host_only(lib):
    from lm_head_linear_03_b200 import flce
    p = flce.plan(8192, 4096, 128256)
    assert p.vocab_chunk == 2048 and p.num_chunks == 63
    assert 1 <= p.lse_splits <= 64
    assert p.launches == 6  # prep, row order, pass 1, combine, pass 2, dX scatter
    assert p.workspace_bytes == flce.workspace_size(8192, 4096, 128256)
    assert p.workspace_reorder_bytes == flce.workspace_size_reorder(8192, 4096)


def test_argument_errors_before_any_launch(lib):
    """NULL pointers and bad sizes are rejected on the host, so these calls are
    safe without a device."""
    i64 = ctypes.c_int64
    f = ctypes.c_float(0)
    assert lib.flce_forward_backward(None, None, None, i64(8), i64(8), i64(8), -100, ctypes.byref(f),
                                     None, None, None, None) == 1
    fake = ctypes.c_void_p(1 << 20)
    assert lib.flce_forward_backward(fake, fake, fake, i64(8), i64(12), i64(8), -100, ctypes.byref(f),
                                     fake, fake, fake, None) == 2  # H % 8
    assert lib.flce_forward_backward(fake, fake, fake, i64(0), i64(8), i64(8), -100, ctypes.byref(f),
                                     fake, fake, fake, None) == 1
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert lib.flce_forward_backward(odd, fake, fake, i64(8), i64(8), i64(8), -100, ctypes.byref(f),
                                     fake, fake, fake, None) == 2  # misaligned X
    r, n = ctypes.c_int32(0), ctypes.c_int32(0)
    assert lib.flce_row_order_info(None, ctypes.byref(r), ctypes.byref(n), None) == 1
    # vocabulary shards: a shard reaching past the vocabulary, or no statistics
    lib.flce_vp_shard_stats.restype = ctypes.c_int
    assert lib.flce_vp_shard_stats(fake, fake, fake, i64(8), i64(8), i64(8), i64(5), i64(10), -100, fake, fake, fake,
                                   fake, ctypes.c_size_t(1 << 30), None) == 1
    assert lib.flce_vp_backward(fake, fake, fake, i64(8), i64(8), i64(8), i64(0), i64(10), -100, 2, None, fake,
                                None, fake, fake, fake, fake, fake, ctypes.c_size_t(1 << 30), None) == 1
    assert lib.flce_row_order_info(odd, ctypes.byref(r), ctypes.byref(n), None) == 1  # misaligned workspace


def _reorder_rule(valid):
    """The row-order rule as the header states it: reorder when the valid rows,
    packed first, fill fewer 256-row tiles than the tiles holding a valid row."""
    import math
    tiles = [sum(valid[i:i + 256]) for i in range(0, len(valid), 256)]
    return math.ceil(sum(valid) / 256) < sum(1 for t in tiles if t)


def test_row_order_rule_on_the_workloads(lib):
    """Which of the named workloads take the reordered path with the workspace
    the benchmark gives them: the rule must say so and the packed-X area must
    fit the 5% budget (host mirror of the device rule; the GPU tests check the
    device)."""
    import torch
    from lm_head_linear_03_b200 import flce
    from lm_head_linear_03_b200.inputs import WORKLOADS, make_targets
    expect = {"tiny": False, "llama3_8b_head": False, "long_context": False,
              "gemma2_large_vocab": True, "phi3_mini_small_vocab": False}
    for name, want in expect.items():
        w = WORKLOADS[name]
        y = make_targets(w, torch.Generator().manual_seed(w.seed))
        has_area = flce.reorder_fits(w.N, w.H, w.V)
        assert (_reorder_rule((y != -100).tolist()) and has_area) == want, name


def test_binding_checks_outputs_before_any_call(lib):
    """The binding rejects, on the host, output buffers of the wrong shape,
    dtype or layout and tensors spread over several devices, before it hands
    any pointer to the library."""
    import torch
    from lm_head_linear_03_b200 import flce
    X = torch.zeros(16, 8, dtype=torch.bfloat16)
    W = torch.zeros(32, 8, dtype=torch.bfloat16)
    y = torch.zeros(16, dtype=torch.int32)
    flce._check_tensors(X, W, y, torch.empty_like(X), torch.empty_like(W), require_cuda=False)
    bad = [
        dict(dX=torch.empty(15, 8, dtype=torch.bfloat16)),                 # too few rows
        dict(dX=torch.empty(16, 8, dtype=torch.float32)),                  # wrong dtype
        dict(dW=torch.empty(8, 32, dtype=torch.bfloat16).t()),             # not contiguous
        dict(dW=torch.empty(33, 8, dtype=torch.bfloat16)),                 # wrong vocabulary size
        dict(workspace=torch.empty(64, dtype=torch.int32)),                # workspace not bytes
        dict(dX=torch.empty(16, 8, dtype=torch.bfloat16, device="meta")),  # another device
    ]
    for kw in bad:
        with pytest.raises(ValueError):
            flce._check_tensors(X, W, y, require_cuda=False, **kw)
    with pytest.raises(ValueError, match="CUDA"):
        flce.forward_backward(X, W, y)
    with pytest.raises(ValueError, match="dX"):
        flce.forward_backward(X, W, y, dX=torch.empty(15, 8, dtype=torch.bfloat16))


def test_noalloc_limit_is_the_base_size(lib):
    """The allocation-free entry takes any problem whose flce_workspace_size fits
    its fixed scratch, even when the reorder workspace does not (it then keeps
    the caller's row order); larger ones are rejected on the host."""
    from lm_head_linear_03_b200 import flce
    N, H, V = 1000, 4096, 256000
    assert flce.workspace_size(N, H, V) <= flce.NOALLOC_SCRATCH_BYTES < flce.workspace_size_reorder(N, H)
    assert flce.workspace_size(2000, 4096, V) > flce.NOALLOC_SCRATCH_BYTES
    i64 = ctypes.c_int64
    f = ctypes.c_float(0)
    fake = ctypes.c_void_p(1 << 20)
    # too large: rejected before the library looks at the device or the pointers
    assert lib.flce_forward_backward_noalloc(fake, fake, fake, i64(2000), i64(4096), i64(V), -100, ctypes.byref(f),
                                             fake, fake, None) == 3
