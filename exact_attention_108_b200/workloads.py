"""Seeded synthetic workloads shared by the tests, the bench and the oracle checks.

This module holds no attention arithmetic: it only names the five workloads and
draws their inputs.  Recipe (the same for every consumer):

* ``g = torch.Generator("cpu").manual_seed(seed)``;
* draw, in this order, Q, K, V and (when wanted) dO as float32 tensors of shape
  [B, H, N, d] with ``torch.randn`` / ``torch.rand`` on ``g``;
* round each to bfloat16 (round-to-nearest-even) -- the GPU consumes these bf16
  tensors and the oracle consumes their exact float64 copies.

The "peaked" distribution (used by the N=8192 stress workload) draws
Q, K ~ 4 * N(0, 1) so that scale * q.k reaches |s| ~ 100, and V ~ U(-1, 1);
dO stays N(0, 1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    dist: str  # "normal" | "peaked"
    backward: bool

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def shape(self):
        return (self.B, self.H, self.N, self.d)

    def fwd_flops(self) -> float:
        """4*B*H*N^2*d, halved when causal (the convention the metric uses)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Backward counted as 2.5x the forward."""
        return 2.5 * self.fwd_flops()


# The five workloads: tiny correctness case; d=64 forward (both mask modes);
# the d=128 causal training shape; the peaked-softmax stress case; long sequence.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 128, 64, False, 0, "normal", True),
    "fwd_d64": Workload("fwd_d64", 8, 16, 2048, 64, False, 1, "normal", False),
    "fwd_d64_causal": Workload("fwd_d64_causal", 8, 16, 2048, 64, True, 1, "normal", False),
    "train_d128_causal": Workload("train_d128_causal", 4, 32, 4096, 128, True, 2, "normal", True),
    "peaked_n8192": Workload("peaked_n8192", 2, 16, 8192, 128, False, 3, "peaked", True),
    "long_n32768_causal": Workload("long_n32768_causal", 1, 8, 32768, 128, True, 4, "normal", True),
}


def make_inputs(B: int, H: int, N: int, d: int, seed: int, dist: str = "normal",
                with_do: bool = True):
    """Return (q, k, v, do) as CPU bfloat16 tensors [B, H, N, d] (do may be None)."""
    g = torch.Generator("cpu").manual_seed(seed)
    shape = (B, H, N, d)
    if dist == "normal":
        q = torch.randn(shape, generator=g, dtype=torch.float32)
        k = torch.randn(shape, generator=g, dtype=torch.float32)
        v = torch.randn(shape, generator=g, dtype=torch.float32)
    elif dist == "peaked":
        q = 4.0 * torch.randn(shape, generator=g, dtype=torch.float32)
        k = 4.0 * torch.randn(shape, generator=g, dtype=torch.float32)
        v = 2.0 * torch.rand(shape, generator=g, dtype=torch.float32) - 1.0
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    do = torch.randn(shape, generator=g, dtype=torch.float32) if with_do else None
    cast = lambda t: None if t is None else t.to(torch.bfloat16)  # noqa: E731
    return cast(q), cast(k), cast(v), cast(do)


def workload_inputs(w: Workload, with_do: bool | None = None):
    if with_do is None:
        with_do = w.backward
    return make_inputs(w.B, w.H, w.N, w.d, w.seed, w.dist, with_do)


def to_f64(t):
    """Exact float64 numpy copy of a (CPU or CUDA) bf16 tensor."""
    return t.detach().to("cpu").to(torch.float64).numpy()
