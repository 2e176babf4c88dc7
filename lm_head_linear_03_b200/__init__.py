"""Fused linear + cross-entropy head for NVIDIA B200 (sm_100a).

``forward_backward(X, W, y)`` returns the token-mean cross-entropy of
``X @ W.T`` against ``y`` (ignore_index -100) together with dX and dW, computed
by hand-written tcgen05/TMA kernels without allocating the N x V logits.  The C
ABI is declared in ``include/flce.h``; ``flce.py`` is its ctypes binding.
"""
from .flce import (  # noqa: F401
    FlceError,
    alloc_workspace,
    count_valid,
    cross_entropy,
    forward_backward,
    forward_backward_async,
    forward_backward_ex,
    forward_backward_host,
    forward_backward_sections,
    load_library,
    pairwise_logistic,
    plan,
    profile_enable,
    profile_read,
    profile_timeline,
    reorder_fits,
    row_order_info,
    vp_backward,
    vp_shard_stats,
    workspace_size,
    workspace_size_reorder,
)
