"""Exact IO-aware attention (forward and backward) for B200 / sm_100a.

The compute runs in ``libfa.so`` (hand-written CUDA for sm_100a behind a C
ABI, declared in ``include/fa.h``). :mod:`exact_io_aware_56_b200.fa` is the
thin ctypes binding with the same entry-point names; it raises if the library
is missing or no CUDA device is present, and there is no CPU fallback.
"""

from .inputs import (  # noqa: F401
    DECODE_WORKLOADS,
    FP8_WORKLOADS,
    WORKLOADS,
    DecodeWorkload,
    Workload,
    make_decode_inputs,
    make_inputs,
    sample_rows,
    to_f64,
    workload_inputs,
)

__all__ = ["DECODE_WORKLOADS", "FP8_WORKLOADS", "WORKLOADS", "DecodeWorkload", "Workload", "make_decode_inputs", "make_inputs",
           "sample_rows", "to_f64", "workload_inputs"]
