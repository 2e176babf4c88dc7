"""Seeded synthetic inputs for the fused linear + cross-entropy head.

This module only draws random numbers: it holds none of the head's arithmetic.
Both the CUDA path and the fp64 oracle are fed from it, so that they see the
same bytes.

The workloads follow the shapes the Liger-Kernel pages talk about: hidden states
``X[N,H]`` and an LM-head weight ``W[V,H]`` in bf16 ("Complete Guide to Liger
Kernel", section LigerFusedLinearCrossEntropyLoss, where the call takes
``(hidden_states, weight, labels)`` with ``weight`` of shape ``(vocab, hidden)``),
and integer targets of the same length as the hidden rows.  Every distribution
below is a reading of the workload recipe, stated where it is chosen:

* ``X ~ N(0, 1)`` and ``W ~ N(0, 0.02)`` with 0.02 the standard deviation, both
  drawn in fp32 and rounded to bf16 (round-to-nearest-even, torch's cast).
* uniform targets: ``randint(0, V)``.
* Zipf(s) targets: ``P(k) ∝ (k+1)^-s`` over ``k = 0..V-1``, drawn by inverse CDF
  from uniform fp64 variates.
* "p% ignored": exactly ``floor(p*N)`` positions, picked by a seeded
  permutation, set to ``ignore_index``; "first P positions ignored": rows
  ``0..P-1``.
"""
from __future__ import annotations

import dataclasses
import math

import torch

IGNORE_INDEX = -100


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic FLCE problem: sizes plus the target recipe."""

    name: str
    N: int
    H: int
    V: int
    targets: str = "uniform"          # "uniform" | "zipf"
    zipf_s: float = 1.1
    ignore_frac: float = 0.0          # fraction of rows set to ignore_index
    ignore_prefix: int = 0            # rows 0..ignore_prefix-1 set to ignore_index
    x_std: float = 1.0
    w_std: float = 0.02
    seed: int = 0

    @property
    def n_ignored(self) -> int:
        return self.ignore_prefix + int(math.floor(self.ignore_frac * self.N))

    def flops(self) -> int:
        """8*N*H*V: forward GEMM, pass-2 recompute, dX and dW contractions."""
        return 8 * self.N * self.H * self.V


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny", N=256, H=256, V=4096, ignore_frac=0.10),
        Workload("llama3_8b_head", N=8192, H=4096, V=128256),
        Workload("long_context", N=16384, H=4096, V=128256, targets="zipf",
                 zipf_s=1.1, ignore_prefix=2048),
        Workload("gemma2_large_vocab", N=4096, H=2304, V=256000, ignore_frac=0.25),
        Workload("phi3_mini_small_vocab", N=32768, H=3072, V=32064, ignore_frac=0.05),
    )
}


def zipf_targets(n: int, V: int, s: float, gen: torch.Generator) -> torch.Tensor:
    """Inverse-CDF draw of ``n`` ranks from P(k) ∝ (k+1)^-s, k in [0, V)."""
    k = torch.arange(1, V + 1, dtype=torch.float64)
    cdf = torch.cumsum(k.pow(-s), 0)
    cdf = cdf / cdf[-1]
    u = torch.rand(n, dtype=torch.float64, generator=gen)
    idx = torch.searchsorted(cdf, u, right=True)
    return idx.clamp_(max=V - 1).to(torch.int32)


def make_targets(w: Workload, gen: torch.Generator, ignore_index: int = IGNORE_INDEX) -> torch.Tensor:
    if w.targets == "uniform":
        y = torch.randint(0, w.V, (w.N,), generator=gen, dtype=torch.int64).to(torch.int32)
    elif w.targets == "zipf":
        y = zipf_targets(w.N, w.V, w.zipf_s, gen)
    else:
        raise ValueError(f"unknown target recipe {w.targets!r}")
    if w.ignore_prefix:
        y[: w.ignore_prefix] = ignore_index
    n_frac = int(math.floor(w.ignore_frac * w.N))
    if n_frac:
        pos = torch.randperm(w.N, generator=gen)[:n_frac]
        y[pos] = ignore_index
    return y


def make_inputs(w: Workload, device: str | torch.device = "cpu", ignore_index: int = IGNORE_INDEX):
    """Returns ``(X bf16[N,H], W bf16[V,H], y int32[N])`` for workload ``w``.

    The draws happen on ``device`` with a generator seeded by ``w.seed``; CPU and
    CUDA generators give different streams, so parity checks draw on the CPU and
    copy the bytes.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device).manual_seed(w.seed)
    X = torch.randn(w.N, w.H, generator=gen, device=device, dtype=torch.float32)
    if w.x_std != 1.0:
        X.mul_(w.x_std)
    X = X.to(torch.bfloat16)
    Wt = torch.randn(w.V, w.H, generator=gen, device=device, dtype=torch.float32)
    Wt.mul_(w.w_std)
    Wt = Wt.to(torch.bfloat16)
    cpu_gen = gen if device.type == "cpu" else torch.Generator().manual_seed(w.seed + 1)
    y = make_targets(w, cpu_gen, ignore_index).to(device)
    return X, Wt, y


def custom(name: str, N: int, H: int, V: int, **kw) -> Workload:
    """A workload with explicit sizes (parity cases, edge shapes)."""
    return Workload(name, N=N, H=H, V=V, **kw)
