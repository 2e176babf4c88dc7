"""ctypes binding of the FLCE C ABI (include/flce.h).

Argument marshalling only: every step of the computation runs in the CUDA
library ``_lib/libflce.so``.  PyTorch supplies device memory and streams.  If the
library is missing, or the device is not sm_100, calls raise; there is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libflce.so")

FLCE_OK = 0
STATUS_NAMES = {
    0: "FLCE_OK",
    1: "FLCE_ERR_INVALID_ARGUMENT",
    2: "FLCE_ERR_UNSUPPORTED",
    3: "FLCE_ERR_WORKSPACE_TOO_SMALL",
    4: "FLCE_ERR_TARGET_OUT_OF_RANGE",
    5: "FLCE_ERR_TIMEOUT",
    6: "FLCE_ERR_CUDA",
}
NUM_KERNEL_KINDS = 8

EXPORTED = (
    "flce_status_string",
    "flce_last_cuda_error",
    "flce_workspace_size",
    "flce_workspace_size_reorder",
    "flce_forward_backward",
    "flce_forward_backward_async",
    "flce_forward_backward_host",
    "flce_plan",
    "flce_kernel_name",
    "flce_profile_enable",
    "flce_profile_read",
    "flce_profile_timeline",
    "flce_forward_backward_noalloc",
    "flce_forward_backward_ex",
    "flce_ce_workspace_size",
    "flce_cross_entropy",
    "flce_probe_bounded_wait",
    "flce_probe_pass2_timeout",
    "flce_row_order_info",
    "flce_vp_shard_stats",
    "flce_vp_backward",
    "flce_count_valid",
    "flce_pairwise_logistic",
    "flce_forward_backward_sections",
)
REDUCTIONS = {"mean": 0, "sum": 1, "none": 2}
NOALLOC_SCRATCH_BYTES = 16 << 20


class FlceError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {STATUS_NAMES.get(status, status)}"
        if status == 6 and _lib is not None:  # FLCE_ERR_CUDA: say which step failed and why
            line, code, text = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_char_p()
            _lib.flce_last_cuda_error(ctypes.byref(line), ctypes.byref(code), ctypes.byref(text))
            msg += f" (library line {line.value}: CUDA error {code.value}, {(text.value or b'').decode()})"
        super().__init__(msg)


class PlanT(ctypes.Structure):
    _fields_ = [
        ("workspace_bytes", ctypes.c_int64),
        ("workspace_reorder_bytes", ctypes.c_int64),
        ("vocab_chunk", ctypes.c_int32),
        ("num_chunks", ctypes.c_int32),
        ("lse_splits", ctypes.c_int32),
        ("launches", ctypes.c_int32),
        ("num_sms", ctypes.c_int32),
    ]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libflce.so (built by ``__graft_entry__.build()``) and declares the ABI."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"FLCE CUDA library not built: {path} is missing (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
    fp = ctypes.POINTER(ctypes.c_float)
    lib.flce_status_string.argtypes = [ctypes.c_int]
    lib.flce_status_string.restype = ctypes.c_char_p
    lib.flce_last_cuda_error.argtypes = [ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_char_p)]
    lib.flce_last_cuda_error.restype = None
    lib.flce_workspace_size.argtypes = [i64, i64, i64]
    lib.flce_workspace_size.restype = sz
    lib.flce_workspace_size_reorder.argtypes = [i64, i64]
    lib.flce_workspace_size_reorder.restype = sz
    lib.flce_forward_backward.argtypes = [vp, vp, vp, i64, i64, i64, i32, fp, vp, vp, vp, vp]
    lib.flce_forward_backward.restype = ctypes.c_int
    lib.flce_forward_backward_async.argtypes = [vp, vp, vp, i64, i64, i64, i32, vp, vp, vp, vp, vp, sz, vp]
    lib.flce_forward_backward_async.restype = ctypes.c_int
    lib.flce_forward_backward_host.argtypes = [vp, vp, vp, i64, i64, i64, i32, fp, vp, vp,
                                               vp, vp, vp, vp, vp, vp, sz, vp]
    lib.flce_forward_backward_host.restype = ctypes.c_int
    lib.flce_plan.argtypes = [i64, i64, i64, ctypes.POINTER(PlanT)]
    lib.flce_plan.restype = ctypes.c_int
    lib.flce_kernel_name.argtypes = [ctypes.c_int]
    lib.flce_kernel_name.restype = ctypes.c_char_p
    lib.flce_profile_enable.argtypes = [ctypes.c_int]
    lib.flce_profile_enable.restype = ctypes.c_int
    lib.flce_profile_read.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_double)]
    lib.flce_profile_read.restype = ctypes.c_int
    lib.flce_profile_timeline.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_double),
                                          ctypes.POINTER(ctypes.c_double), ctypes.c_int32,
                                          ctypes.POINTER(ctypes.c_int32)]
    lib.flce_profile_timeline.restype = ctypes.c_int
    lib.flce_forward_backward_ex.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                             vp]
    lib.flce_forward_backward_ex.restype = ctypes.c_int
    lib.flce_ce_workspace_size.argtypes = [i64, i64]
    lib.flce_ce_workspace_size.restype = sz
    lib.flce_cross_entropy.argtypes = [vp, vp, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.flce_cross_entropy.restype = ctypes.c_int
    lib.flce_probe_bounded_wait.argtypes = [i64, vp, vp]
    lib.flce_probe_bounded_wait.restype = ctypes.c_int
    lib.flce_probe_pass2_timeout.argtypes = [vp, vp, vp, i64, i64, i64, i32, vp, vp, vp, vp, vp, sz, i64, vp]
    lib.flce_probe_pass2_timeout.restype = ctypes.c_int
    lib.flce_forward_backward_noalloc.argtypes = [vp, vp, vp, i64, i64, i64, i32, fp, vp, vp, vp]
    lib.flce_forward_backward_noalloc.restype = ctypes.c_int
    lib.flce_row_order_info.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(i32), vp]
    lib.flce_row_order_info.restype = ctypes.c_int
    lib.flce_vp_shard_stats.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i32, vp, vp, vp, vp, sz, vp]
    lib.flce_vp_shard_stats.restype = ctypes.c_int
    lib.flce_vp_backward.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp,
                                     vp, sz, vp]
    lib.flce_vp_backward.restype = ctypes.c_int
    lib.flce_forward_backward_sections.argtypes = [vp, vp, vp, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, sz, i32,
                                                   ctypes.POINTER(vp), ctypes.POINTER(i64), vp]
    lib.flce_forward_backward_sections.restype = ctypes.c_int
    lib.flce_count_valid.argtypes = [vp, i64, i32, vp, vp]
    lib.flce_count_valid.restype = ctypes.c_int
    lib.flce_pairwise_logistic.argtypes = [vp, vp, i64, i32, vp, i32, vp, vp, i32, ctypes.c_double, vp, vp, vp, vp,
                                           vp, vp, vp]
    lib.flce_pairwise_logistic.restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != FLCE_OK:
        raise FlceError(status, where)


def _stream_handle(stream, device=None):
    """The raw handle of ``stream``, or of the current stream of ``device``."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _check_tensors(X, W, y, dX=None, dW=None, workspace=None, require_cuda=True):
    """X bf16 [N,H], W bf16 [V,H], y int32 [N], optional outputs dX bf16 [N,H]
    and dW bf16 [V,H] and a uint8 workspace: all contiguous and on one device,
    a CUDA device unless ``require_cuda`` is False.  Raises ValueError."""
    if X.dtype != torch.bfloat16 or W.dtype != torch.bfloat16 or y.dtype != torch.int32:
        raise ValueError("expected X, W bf16 and y int32")
    if X.dim() != 2 or W.dim() != 2 or y.dim() != 1:
        raise ValueError("expected X[N,H], W[V,H], y[N]")
    if X.shape[1] != W.shape[1] or y.shape[0] != X.shape[0]:
        raise ValueError(f"shape mismatch: X{tuple(X.shape)} W{tuple(W.shape)} y{tuple(y.shape)}")
    if not (X.is_contiguous() and W.is_contiguous() and y.is_contiguous()):
        raise ValueError("X, W and y must be contiguous")
    for name, t, like in (("dX", dX, X), ("dW", dW, W)):
        if t is None:
            continue
        if t.dtype != torch.bfloat16 or tuple(t.shape) != tuple(like.shape) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor of shape {tuple(like.shape)}, "
                             f"got {t.dtype} {tuple(t.shape)}")
    if workspace is not None and (workspace.dtype != torch.uint8 or workspace.dim() != 1
                                  or not workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous 1-D uint8 tensor")
    devices = {t.device for t in (X, W, y, dX, dW, workspace) if t is not None}
    if len(devices) != 1:
        raise ValueError(f"all tensors of a call must be on one device, got {sorted(map(str, devices))}")
    if require_cuda and X.device.type != "cuda":
        raise ValueError("X, W and y must be CUDA tensors")


def _check_inputs(X, W, y):
    _check_tensors(X, W, y)


def workspace_size(N: int, H: int, V: int = 1) -> int:
    """flce_workspace_size: bytes one call needs; independent of V."""
    return int(load_library().flce_workspace_size(N, H, V))


def workspace_size_reorder(N: int, H: int) -> int:
    """flce_workspace_size_reorder: bytes of a workspace that also holds the
    packed copy of X, so that scattered ignored rows can be skipped."""
    return int(load_library().flce_workspace_size_reorder(N, H))


def plan(N: int, H: int, V: int) -> PlanT:
    p = PlanT()
    _check(load_library().flce_plan(N, H, V, ctypes.byref(p)), "flce_plan")
    return p


def packed_x_bytes(N: int, H: int) -> int:
    """Size of the workspace area for the packed copy of X: N x H bf16, rounded
    up to 256 bytes."""
    return (N * H * 2 + 255) // 256 * 256


def reorder_fits(N: int, H: int, V: int, budget: float = 0.05) -> bool:
    """Whether a workspace with the packed-X area stays within ``budget`` of the
    N x V bf16 logit tensor that the head never stores (5% is the bound the
    workload specification sets).  The benchmark and the full-size tests use it
    to choose the workspace; the library itself takes whatever it is given."""
    return workspace_size_reorder(N, H) <= budget * 2.0 * N * V


def alloc_workspace(N: int, H: int, V: int = 1, device=None, reorder: bool = False) -> torch.Tensor:
    """A uint8 device buffer for one call (torch's allocator hands out 512-B
    aligned blocks): flce_workspace_size bytes, or flce_workspace_size_reorder
    bytes with ``reorder`` (then scattered ignored rows can be skipped).  V does
    not change the size."""
    nbytes = workspace_size_reorder(N, H) if reorder else workspace_size(N, H, V)
    return torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")


def _check_aux(t, dtype, numel, device, name):
    """A small device buffer of the call (loss, status, per-row vectors):
    contiguous, of ``dtype`` and at least ``numel`` elements, on ``device``."""
    if t is None:
        return
    if t.dtype != dtype or not t.is_contiguous() or t.numel() < numel or t.device != device:
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of {numel} elements on {device}")


def row_order_info(workspace: torch.Tensor, stream=None):
    """(reordered, n_valid) of the last call that used ``workspace``: whether its
    token rows were reordered (valid rows first, X packed in that order) and
    how many rows had a non-ignored target.  Waits for ``stream``."""
    r, n = ctypes.c_int32(0), ctypes.c_int32(0)
    with torch.cuda.device(workspace.device):
        _check(load_library().flce_row_order_info(_ptr(workspace), ctypes.byref(r), ctypes.byref(n),
                                                  _stream_handle(stream, workspace.device)), "flce_row_order_info")
    return bool(r.value), int(n.value)


def forward_backward(X, W, y, ignore_index: int = -100, *, dX=None, dW=None, workspace=None, stream=None):
    """Synchronous call: returns (loss: float, dX, dW).  Raises FlceError on any
    host- or device-detected error."""
    lib = load_library()
    _check_tensors(X, W, y, dX, dW, workspace)
    N, H = X.shape
    V = W.shape[0]
    dX = torch.empty_like(X) if dX is None else dX
    dW = torch.empty_like(W) if dW is None else dW
    workspace = alloc_workspace(N, H, V, X.device) if workspace is None else workspace
    if workspace.numel() < workspace_size(N, H, V):
        raise ValueError("workspace smaller than flce_workspace_size")
    loss = ctypes.c_float(0.0)
    with torch.cuda.device(X.device):
        st = lib.flce_forward_backward(_ptr(X), _ptr(W), _ptr(y), N, H, V, ignore_index, ctypes.byref(loss),
                                       _ptr(dX), _ptr(dW), _ptr(workspace), _stream_handle(stream, X.device))
    _check(st, "flce_forward_backward")
    return loss.value, dX, dW


def forward_backward_async(X, W, y, ignore_index: int = -100, *, out=None, workspace=None, stream=None):
    """Enqueues the call and returns device tensors (loss[1] f32, status[1] i32, dX, dW)
    without waiting.  ``out`` may pass preallocated (loss, status, dX, dW)."""
    lib = load_library()
    N, H = X.shape
    V = W.shape[0]
    if out is None:
        out = (torch.empty(1, dtype=torch.float32, device=X.device),
               torch.empty(1, dtype=torch.int32, device=X.device),
               torch.empty_like(X), torch.empty_like(W))
    loss, status, dX, dW = out
    _check_tensors(X, W, y, dX, dW, workspace)
    _check_aux(loss, torch.float32, 1, X.device, "loss")
    _check_aux(status, torch.int32, 1, X.device, "status")
    workspace = alloc_workspace(N, H, V, X.device) if workspace is None else workspace
    with torch.cuda.device(X.device):
        st = lib.flce_forward_backward_async(_ptr(X), _ptr(W), _ptr(y), N, H, V, ignore_index, _ptr(loss),
                                             _ptr(status), _ptr(dX), _ptr(dW), _ptr(workspace),
                                             workspace.numel(), _stream_handle(stream, X.device))
    _check(st, "flce_forward_backward_async")
    return loss, status, dX, dW


def forward_backward_ex(X, W, y, ignore_index: int = -100, *, reduction: str = "mean", grad_row_scale=None,
                        mean_count=None, row_loss: bool = False, grads: bool = True, workspace=None, stream=None):
    """Asynchronous call with every option; returns device tensors
    (loss[1], status[1], row_loss[N] or None, dX or None, dW or None).

    reduction 'mean' | 'sum' | 'none'; grad_row_scale: fp32[N] upstream
    gradient of each row's loss for 'none'; mean_count: int32[1] device count
    the mean divides by instead of this call's n_valid; grads=False skips the
    gradient pass.
    """
    lib = load_library()
    _check_tensors(X, W, y, workspace=workspace)
    N, H = X.shape
    V = W.shape[0]
    dev = X.device
    _check_aux(grad_row_scale, torch.float32, N, dev, "grad_row_scale")
    _check_aux(mean_count, torch.int32, 1, dev, "mean_count")
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    status = torch.empty(1, dtype=torch.int32, device=dev)
    rl = torch.empty(N, dtype=torch.float32, device=dev) if row_loss else None
    dX = torch.empty_like(X) if grads else None
    dW = torch.empty_like(W) if grads else None
    workspace = alloc_workspace(N, H, V, dev) if workspace is None else workspace
    vp = lambda t: None if t is None else _ptr(t)  # noqa: E731
    with torch.cuda.device(dev):
        st = lib.flce_forward_backward_ex(_ptr(X), _ptr(W), _ptr(y), N, H, V, ignore_index, REDUCTIONS[reduction],
                                          vp(grad_row_scale), vp(mean_count), _ptr(loss), vp(rl), _ptr(status),
                                          vp(dX), vp(dW), _ptr(workspace), workspace.numel(),
                                          _stream_handle(stream, dev))
    _check(st, "flce_forward_backward_ex")
    return loss, status, rl, dX, dW


def vp_shard_stats(X, W_shard, y, v0: int, V: int, ignore_index: int = -100, *, workspace=None, stream=None):
    """Step 1 of the vocabulary-parallel head on this rank's shard, W rows
    ``[v0, v0 + W_shard.shape[0])`` of a ``V``-entry vocabulary.  Returns device
    tensors (shard_lse[N], shard_zy[N], status[1]) without waiting."""
    lib = load_library()
    _check_tensors(X, W_shard, y, workspace=workspace)
    N, H = X.shape
    Vs = W_shard.shape[0]
    dev = X.device
    lse = torch.empty(N, dtype=torch.float32, device=dev)
    zy = torch.empty(N, dtype=torch.float32, device=dev)
    status = torch.empty(1, dtype=torch.int32, device=dev)
    workspace = alloc_workspace(N, H, 1, dev) if workspace is None else workspace
    with torch.cuda.device(dev):
        st = lib.flce_vp_shard_stats(_ptr(X), _ptr(W_shard), _ptr(y), N, H, Vs, v0, V, ignore_index, _ptr(lse),
                                     _ptr(zy), _ptr(status), _ptr(workspace), workspace.numel(),
                                     _stream_handle(stream, dev))
    _check(st, "flce_vp_shard_stats")
    return lse, zy, status


def vp_backward(X, W_shard, y, v0: int, V: int, all_lse, all_zy, ignore_index: int = -100, *, mean_count=None,
                grads: bool = True, workspace=None, stream=None):
    """Step 3 of the vocabulary-parallel head: every shard's statistics
    (``all_lse``, ``all_zy``: float32 [shards][N]) give the loss; returns device
    tensors (loss[1], status[1], dX_part or None, dW_shard or None) without
    waiting.  dX_part is this shard's share of dX (sum it over the ranks)."""
    lib = load_library()
    _check_tensors(X, W_shard, y, workspace=workspace)
    N, H = X.shape
    Vs = W_shard.shape[0]
    dev = X.device
    for t in (all_lse, all_zy):
        if t.dtype != torch.float32 or t.device != dev or t.dim() != 2 or t.shape[1] != N or not t.is_contiguous():
            raise ValueError(f"all_lse / all_zy must be contiguous float32 tensors of shape [shards, N] on {dev}")
    if all_lse.shape != all_zy.shape:
        raise ValueError("all_lse and all_zy differ in shape")
    _check_aux(mean_count, torch.int32, 1, dev, "mean_count")
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    status = torch.empty(1, dtype=torch.int32, device=dev)
    dX = torch.empty_like(X) if grads else None
    dW = torch.empty_like(W_shard) if grads else None
    workspace = alloc_workspace(N, H, 1, dev) if workspace is None else workspace
    vp = lambda t: None if t is None else _ptr(t)  # noqa: E731
    with torch.cuda.device(dev):
        st = lib.flce_vp_backward(_ptr(X), _ptr(W_shard), _ptr(y), N, H, Vs, v0, V, ignore_index, all_lse.shape[0],
                                  _ptr(all_lse), _ptr(all_zy), vp(mean_count), _ptr(loss), _ptr(status), vp(dX),
                                  vp(dW), _ptr(workspace), workspace.numel(), _stream_handle(stream, dev))
    _check(st, "flce_vp_backward")
    return loss, status, dX, dW


def cross_entropy(logits, y, ignore_index: int = -100, *, reduction: str = "mean", grad_row_scale=None,
                  row_loss: bool = False, grad: str = "new", workspace=None, stream=None):
    """Cross-entropy on given bf16 logits [N, V]; asynchronous.  Returns device
    tensors (loss[1], status[1], row_loss[N] or None, dlogits or None).
    grad: 'new' (a new tensor), 'inplace' (overwrite ``logits``) or 'none'."""
    lib = load_library()
    if not (logits.is_cuda and y.is_cuda) or logits.dtype != torch.bfloat16 or y.dtype != torch.int32:
        raise ValueError("expected CUDA bf16 logits and int32 targets")
    if logits.dim() != 2 or y.shape != (logits.shape[0],) or not (logits.is_contiguous() and y.is_contiguous()):
        raise ValueError("expected contiguous logits [N, V] and targets [N]")
    N, V = logits.shape
    dev = logits.device
    if y.device != dev or (workspace is not None and workspace.device != dev):
        raise ValueError("logits, targets and workspace must be on one device")
    _check_aux(grad_row_scale, torch.float32, N, dev, "grad_row_scale")
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    status = torch.empty(1, dtype=torch.int32, device=dev)
    rl = torch.empty(N, dtype=torch.float32, device=dev) if row_loss else None
    dz = {"new": lambda: torch.empty_like(logits), "inplace": lambda: logits, "none": lambda: None}[grad]()
    if workspace is None:
        workspace = torch.empty(int(lib.flce_ce_workspace_size(N, V)), dtype=torch.uint8, device=dev)
    vp = lambda t: None if t is None else _ptr(t)  # noqa: E731
    with torch.cuda.device(dev):
        st = lib.flce_cross_entropy(_ptr(logits), _ptr(y), N, V, ignore_index, REDUCTIONS[reduction],
                                    vp(grad_row_scale), _ptr(loss), vp(rl), _ptr(status), vp(dz), _ptr(workspace),
                                    workspace.numel(), _stream_handle(stream, dev))
    _check(st, "flce_cross_entropy")
    return loss, status, rl, dz


def forward_backward_host(hX, hW, hy, dev_bufs, ignore_index: int = -100, *, h_out=None, stream=None):
    """End-to-end call on host tensors: copies in, computes, copies loss, dX and
    dW back.  ``dev_bufs`` = (d_X, d_W, d_y, d_dX, d_dW, workspace) on the device;
    ``h_out`` = optional host (dX, dW) outputs (pinned for full bandwidth)."""
    lib = load_library()
    N, H = hX.shape
    V = hW.shape[0]
    d_X, d_W, d_y, d_dX, d_dW, ws = dev_bufs
    if h_out is None:
        h_out = (torch.empty_like(hX), torch.empty_like(hW))
    h_dX, h_dW = h_out
    _check_tensors(hX, hW, hy, h_dX, h_dW, require_cuda=False)
    if hX.device.type != "cpu":
        raise ValueError("hX, hW, hy and the host outputs must be CPU tensors")
    _check_tensors(d_X, d_W, d_y, d_dX, d_dW, ws)
    if d_X.shape != hX.shape or d_W.shape != hW.shape:
        raise ValueError("device buffers must have the host tensors' shapes")
    loss = ctypes.c_float(0.0)
    with torch.cuda.device(d_X.device):
        st = lib.flce_forward_backward_host(_ptr(hX), _ptr(hW), _ptr(hy), N, H, V, ignore_index,
                                            ctypes.byref(loss), _ptr(h_dX), _ptr(h_dW), _ptr(d_X), _ptr(d_W),
                                            _ptr(d_y), _ptr(d_dX), _ptr(d_dW), _ptr(ws), ws.numel(),
                                            _stream_handle(stream, d_X.device))
    _check(st, "flce_forward_backward_host")
    return loss.value, h_dX, h_dW


def kernel_names():
    lib = load_library()
    return [lib.flce_kernel_name(k).decode() for k in range(NUM_KERNEL_KINDS)]


def profile_enable(on: bool = True):
    _check(load_library().flce_profile_enable(1 if on else 0), "flce_profile_enable")


def profile_read():
    """{kernel name: (launches, total ms)} since the last read."""
    lib = load_library()
    n = (ctypes.c_int32 * NUM_KERNEL_KINDS)()
    ms = (ctypes.c_double * NUM_KERNEL_KINDS)()
    _check(lib.flce_profile_read(n, ms), "flce_profile_read")
    names = kernel_names()
    return {names[k]: (int(n[k]), float(ms[k])) for k in range(NUM_KERNEL_KINDS)}


def profile_timeline(capacity: int = 4096):
    """[(name, begin ms, end ms)] of every recorded launch and host-buffer
    copy since the last read, in record order, relative to the first begin."""
    lib = load_library()
    kinds = (ctypes.c_int32 * capacity)()
    b = (ctypes.c_double * capacity)()
    e = (ctypes.c_double * capacity)()
    n = ctypes.c_int32()
    _check(lib.flce_profile_timeline(kinds, b, e, capacity, ctypes.byref(n)), "flce_profile_timeline")
    return [(lib.flce_kernel_name(kinds[i]).decode(), float(b[i]), float(e[i])) for i in range(min(n.value, capacity))]


def forward_backward_noalloc(X, W, y, ignore_index: int = -100, *, dX=None, dW=None, stream=None):
    """Like :func:`forward_backward` but with no workspace: the library uses its
    fixed device scratch array (NOALLOC_SCRATCH_BYTES), for callers that cannot
    allocate device memory.  Problems whose flce_workspace_size exceeds it raise
    FLCE_ERR_WORKSPACE_TOO_SMALL; overlapping calls race on the shared array.
    The call runs with X's device current, on that device's current stream
    unless ``stream`` is given: the scratch array the library picks is that
    device's."""
    lib = load_library()
    _check_tensors(X, W, y, dX, dW)
    N, H = X.shape
    V = W.shape[0]
    dX = torch.empty_like(X) if dX is None else dX
    dW = torch.empty_like(W) if dW is None else dW
    loss = ctypes.c_float(0.0)
    with torch.cuda.device(X.device):
        st = lib.flce_forward_backward_noalloc(_ptr(X), _ptr(W), _ptr(y), N, H, V, ignore_index,
                                               ctypes.byref(loss), _ptr(dX), _ptr(dW),
                                               _stream_handle(stream, X.device))
    _check(st, "flce_forward_backward_noalloc")
    return loss.value, dX, dW


def probe_pass2_timeout(X, W, y, ignore_index: int = -100, *, timeout_ns: int = 5_000_000, workspace=None,
                        stream=None):
    """Enqueues one call whose pass-2 dW items wait for a tile that never
    comes, every wait bounded by ``timeout_ns``; returns the device status
    tensor int32[1] (FLCE_ERR_TIMEOUT once the stream gets there)."""
    lib = load_library()
    _check_tensors(X, W, y, workspace=workspace)
    N, H = X.shape
    V = W.shape[0]
    loss = torch.empty(1, dtype=torch.float32, device=X.device)
    status = torch.empty(1, dtype=torch.int32, device=X.device)
    dX, dW = torch.empty_like(X), torch.empty_like(W)
    workspace = alloc_workspace(N, H, V, X.device) if workspace is None else workspace
    with torch.cuda.device(X.device):
        _check(lib.flce_probe_pass2_timeout(_ptr(X), _ptr(W), _ptr(y), N, H, V, ignore_index, _ptr(loss),
                                            _ptr(status), _ptr(dX), _ptr(dW), _ptr(workspace), workspace.numel(),
                                            timeout_ns, _stream_handle(stream, X.device)),
               "flce_probe_pass2_timeout")
    return status


def probe_bounded_wait(timeout_ns: int = 1_000_000, stream=None, device=None):
    """Runs the bounded-wait probe and returns its device status tensor int32[3]."""
    lib = load_library()
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    st = torch.empty(3, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib.flce_probe_bounded_wait(timeout_ns, _ptr(st), _stream_handle(stream, dev)),
               "flce_probe_bounded_wait")
    return st


def count_valid(y, ignore_index: int = -100, *, out=None, stream=None):
    """flce_count_valid: the number of targets != ignore_index, as a device
    int32[1] tensor (asynchronous)."""
    lib = load_library()
    if y.dtype != torch.int32 or y.dim() != 1 or not y.is_contiguous() or not y.is_cuda:
        raise ValueError("y must be a contiguous CUDA int32 tensor [N]")
    out = torch.empty(1, dtype=torch.int32, device=y.device) if out is None else out
    _check_aux(out, torch.int32, 1, y.device, "out")
    with torch.cuda.device(y.device):
        _check(lib.flce_count_valid(_ptr(y), y.numel(), ignore_index, _ptr(out), _stream_handle(stream, y.device)),
               "flce_count_valid")
    return out


def pairwise_logistic(row_loss, y, seq_start, chosen, rejected, beta: float, ref_logp=None,
                      ignore_index: int = -100, *, stream=None):
    """flce_pairwise_logistic on device tensors: row_loss fp32 [N], y int32 [N],
    seq_start int32 [S+1], chosen / rejected int32 [P], ref_logp fp64 [S] or
    None.  Returns device tensors (loss fp64[1], logp fp64[S], grad_logp
    fp64[S], row_weight fp32[N], status int32[1]) without waiting."""
    lib = load_library()
    dev = row_loss.device
    N = row_loss.numel()
    S = seq_start.numel() - 1
    P = chosen.numel()
    _check_aux(row_loss, torch.float32, N, dev, "row_loss")
    _check_aux(y, torch.int32, N, dev, "y")
    _check_aux(seq_start, torch.int32, S + 1, dev, "seq_start")
    _check_aux(chosen, torch.int32, P, dev, "chosen")
    _check_aux(rejected, torch.int32, P, dev, "rejected")
    _check_aux(ref_logp, torch.float64, S, dev, "ref_logp")
    if not row_loss.is_cuda or rejected.numel() != P or y.numel() != N:
        raise ValueError("expected CUDA tensors, y[N] beside row_loss[N] and as many rejected as chosen ids")
    loss = torch.empty(1, dtype=torch.float64, device=dev)
    logp = torch.empty(S, dtype=torch.float64, device=dev)
    grad = torch.empty(S, dtype=torch.float64, device=dev)
    weight = torch.empty(N, dtype=torch.float32, device=dev)
    status = torch.empty(1, dtype=torch.int32, device=dev)
    vp = lambda t: None if t is None else _ptr(t)  # noqa: E731
    with torch.cuda.device(dev):
        _check(lib.flce_pairwise_logistic(_ptr(row_loss), _ptr(y), N, ignore_index, _ptr(seq_start), S,
                                          _ptr(chosen), _ptr(rejected), P, float(beta), vp(ref_logp), _ptr(loss),
                                          _ptr(logp), _ptr(grad), _ptr(weight), _ptr(status),
                                          _stream_handle(stream, dev)), "flce_pairwise_logistic")
    return loss, logp, grad, weight, status


def forward_backward_sections(X, W, y, ignore_index: int = -100, *, sections: int = 4, mean_count=None, out=None,
                              workspace=None, stream=None):
    """flce_forward_backward_sections: the mean-reduced call with the gradient
    pass in ``sections`` launches.  Returns (loss[1], status[1], dX, dW, events,
    rows): ``events[k]`` (torch.cuda.Event) completes when dW rows
    ``rows[k]:rows[k+1]`` are final.  Asynchronous."""
    lib = load_library()
    N, H = X.shape
    V = W.shape[0]
    dev = X.device
    if out is None:
        out = (torch.empty(1, dtype=torch.float32, device=dev), torch.empty(1, dtype=torch.int32, device=dev),
               torch.empty_like(X), torch.empty_like(W))
    loss, status, dX, dW = out
    _check_tensors(X, W, y, dX, dW, workspace)
    _check_aux(loss, torch.float32, 1, dev, "loss")
    _check_aux(status, torch.int32, 1, dev, "status")
    _check_aux(mean_count, torch.int32, 1, dev, "mean_count")
    workspace = alloc_workspace(N, H, V, dev) if workspace is None else workspace
    strm = stream if stream is not None else torch.cuda.current_stream(dev)
    events = [torch.cuda.Event() for _ in range(sections)]
    for e in events:  # the handle exists once the event has been recorded
        e.record(strm)
    handles = (ctypes.c_void_p * sections)(*[e.cuda_event for e in events])
    rows = (ctypes.c_int64 * (sections + 1))()
    vp = lambda t: None if t is None else _ptr(t)  # noqa: E731
    with torch.cuda.device(dev):
        _check(lib.flce_forward_backward_sections(_ptr(X), _ptr(W), _ptr(y), N, H, V, ignore_index, vp(mean_count),
                                                  _ptr(loss), _ptr(status), _ptr(dX), _ptr(dW), _ptr(workspace),
                                                  workspace.numel(), sections, handles, rows,
                                                  ctypes.c_void_p(strm.cuda_stream)),
               "flce_forward_backward_sections")
    return loss, status, dX, dW, events, [int(r) for r in rows]
