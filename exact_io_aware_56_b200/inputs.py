"""Seeded synthetic inputs and the named attention workloads.

This module holds no attention arithmetic: it only draws random numbers and
names shapes. Both the CUDA path's tests and the fp64 oracle consume what it
returns, so that the two see the same bits.

Recipe: q, k, v and dout are drawn in that order from one CPU
``torch.Generator`` seeded with ``seed``, as i.i.d. standard normals in fp32;
q and k are multiplied by ``qk_gain`` (2 for the peaky-row workload, else 1);
all four are rounded to bf16 (round to nearest even). The oracle upcasts those
bf16 values to float64, so a parity error measures the kernel, not the input
rounding.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, masking and input recipe."""

    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    backward: bool
    qk_gain: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def fwd_flops(self) -> float:
        """Two GEMMs of 2*N*N*d flops per head; half of that when causal."""
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Five GEMMs (QK^T recompute, dV, dP, dK, dQ) = 2.5x the forward."""
        return 2.5 * self.fwd_flops() if self.backward else 0.0


# The problems the kernels are checked and timed on. Sizes and value
# distributions are those of the source pages' workloads (synthetic, seeded).
WORKLOADS = {
    w.name: w
    for w in [
        Workload("fwd_b1_h1_n128_d64", 1, 1, 1, 128, 64, False, False, seed=1000),
        Workload("fwdbwd_b4_h16_n2048_d64_causal", 4, 16, 16, 2048, 64, True, True, seed=1001),
        Workload("fwdbwd_b4_h16_n2048_d64", 4, 16, 16, 2048, 64, False, True, seed=1001),
        Workload("fwdbwd_b2_h16_n8192_d128_causal_peaky", 2, 16, 16, 8192, 128, True, True,
                 qk_gain=2.0, seed=1002),
        Workload("fwdbwd_gqa_b1_hq32_hkv8_n16384_d128_causal", 1, 32, 8, 16384, 128, True, True,
                 seed=1003),
        Workload("fwd_b1_h8_n131072_d128_causal", 1, 8, 8, 131072, 128, True, False, seed=1004),
    ]
}


def make_inputs(B, Hq, Hkv, N, d, seed, qk_gain=1.0, with_dout=True):
    """Draw q, k, v (and dout) as bf16 CPU tensors; see the module docstring."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    q = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float32)
    k = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float32)
    if qk_gain != 1.0:
        q.mul_(qk_gain)
        k.mul_(qk_gain)
    out = {
        "q": q.to(torch.bfloat16),
        "k": k.to(torch.bfloat16),
        "v": v.to(torch.bfloat16),
    }
    del q, k, v
    if with_dout:
        out["dout"] = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return out


def workload_inputs(w: Workload, with_dout=None):
    if with_dout is None:
        with_dout = w.backward
    return make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, w.qk_gain, with_dout)


def sample_rows(n: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct row indices in [0, n), drawn from ``seed + 1000``."""
    rng = np.random.default_rng(int(seed) + 1000)
    count = min(count, n)
    return np.sort(rng.choice(n, size=count, replace=False))


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a bf16/fp32 tensor to a float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()
