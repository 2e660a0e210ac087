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


# FP8-mode forward workloads: the same shapes and input recipe as the bf16
# workloads above, quantized to e4m3 (Q, K per 128-row block, V per head)
# before the timed forward.
FP8_WORKLOADS = {
    "fwd_fp8_b2_h16_n8192_d128_causal_peaky": Workload("fwd_fp8_b2_h16_n8192_d128_causal_peaky", 2, 16, 16, 8192,
                                                       128, True, False, qk_gain=2.0, seed=1002),
    "fwd_fp8_gqa_b1_hq32_hkv8_n16384_d128_causal": Workload("fwd_fp8_gqa_b1_hq32_hkv8_n16384_d128_causal", 1, 32,
                                                            8, 16384, 128, True, False, seed=1003),
}


@dataclass(frozen=True)
class DecodeWorkload:
    """Decode against a KV cache: Nq new queries per head, an Nk-key cache.

    Shapes are those of serving a GQA model one token (or a few speculative
    tokens) at a time; the cache is larger than L2, so every call streams it
    from HBM.
    """

    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool = True
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def bytes_moved(self) -> int:
        """Algorithmic HBM bytes of one call: read q, k, v; write o (bf16) and lse (fp32)."""
        qo = 2 * self.B * self.Hq * self.Nq * self.d * 2
        kv = 2 * self.B * self.Hkv * self.Nk * self.d * 2
        return qo + kv + 4 * self.B * self.Hq * self.Nq

    def flops(self) -> float:
        """Two GEMMs of 2*Nq*Nk*d flops per query head (the causal cut is at most Nq^2/2 keys)."""
        return 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.d


DECODE_WORKLOADS = {
    w.name: w
    for w in [
        DecodeWorkload("decode_b16_hq32_hkv8_nq1_nk8192_d128", 16, 32, 8, 1, 8192, 128, seed=1100),
        DecodeWorkload("decode_b4_hq64_hkv8_nq4_nk32768_d128", 4, 64, 8, 4, 32768, 128, seed=1101),
        DecodeWorkload("decode_b64_hq16_hkv16_nq1_nk2048_d64", 64, 16, 16, 1, 2048, 64, seed=1102),
    ]
}


def make_decode_inputs(B, Hq, Hkv, Nq, Nk, d, seed):
    """Draw q [B,Hq,Nq,d] and the cache k, v [B,Hkv,Nk,d] (in that order) as
    bf16 CPU tensors, i.i.d. standard normals rounded from fp32."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    out = {}
    for name, shape in (("q", (B, Hq, Nq, d)), ("k", (B, Hkv, Nk, d)), ("v", (B, Hkv, Nk, d))):
        out[name] = torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return out


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
