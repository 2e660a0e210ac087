"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare with the fp64 oracle on the same bf16 inputs."""

import numpy as np
import torch

from exact_io_aware_56_b200 import fa, make_inputs, to_f64

# Tolerances (from the stated targets): O, dQ, dK, dV max-abs 2e-2 against the
# fp64 oracle; L: |dL| <= 1e-3 * max(1, |L|) (a plain relative bound is
# ill-conditioned where L is near 0).
TOL_ABS = 2e-2
TOL_L = 1e-3


def assert_close_abs(name, got, ref, tol=TOL_ABS):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    err = np.abs(got - ref).max() if got.size else 0.0
    assert err <= tol, f"{name}: max abs err {err:.3e} > {tol:.1e} (max |ref| {np.abs(ref).max():.3e})"
    return err


def assert_close_lse(got, ref, tol=TOL_L):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), "lse: non-finite values"
    err = (np.abs(got - ref) / np.maximum(1.0, np.abs(ref))).max() if got.size else 0.0
    assert err <= tol, f"lse: scaled err {err:.3e} > {tol:.1e}"
    return err


def gpu_inputs(B, Hq, Hkv, N, d, seed, qk_gain=1.0, with_dout=True):
    host = make_inputs(B, Hq, Hkv, N, d, seed, qk_gain, with_dout)
    dev = {k: v.cuda() for k, v in host.items()}
    ref = {k: to_f64(v) for k, v in host.items()}
    return dev, ref


def run_fwd(dev, causal, scale):
    o, lse = fa.attention_forward(dev["q"], dev["k"], dev["v"], causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == fa.FA_OK
    return o, lse
