"""The FMA-pipe exponential of the forward kernel: the committed coefficients
are the ones the committed fitting script produces, and their float32
evaluation stays within the fitted error bound (CPU); on the GPU the device
function agrees with float64 2^x and with the exponential unit's ex2.approx."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from exact_io_aware_56_b200 import fit_exp2_poly as fit

HEADER = fit.HEADER


def header_coeffs(name="C"):
    text = open(HEADER).read()
    vals = dict(re.findall(r"kExp2%s(\d) = (-?0x[0-9a-fp.+-]+)f" % name, text))
    return np.array([float.fromhex(vals[str(k)]) for k in range(len(vals))], dtype=np.float32)


def test_header_matches_fit():
    c, err = fit.fit()
    assert err < 1.2e-4
    np.testing.assert_array_equal(header_coeffs(), c.astype(np.float32))
    assert header_coeffs()[0] == 1.0 and header_coeffs("A")[0] == 1.0


def test_accurate_header_matches_fit():
    c, err = fit.fit(fit.DEGREE_ACCURATE)
    assert err < 1e-8
    np.testing.assert_array_equal(header_coeffs("A"), c.astype(np.float32))


def test_accurate_float32_evaluation_error_bound():
    # The rescale factor's exponential: float32 evaluation within a few
    # float32 rounding steps of 2^x, exact zeros below the range.
    c = header_coeffs("A")
    rng = np.random.default_rng(3)
    x = np.concatenate([-rng.uniform(0, 125, 1_000_000), -rng.uniform(0, 1, 100_000), np.arange(0, -125, -0.25)])
    x = x.astype(np.float32)
    y = fit.eval_f32(c, x)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 5e-7
    assert fit.eval_f32(c, np.array([0.0], dtype=np.float32))[0] == 1.0
    assert (fit.eval_f32(c, np.array([-np.inf, -126.0, -200.0], dtype=np.float32)) == 0).all()


def test_float32_evaluation_error_bound():
    c = header_coeffs()
    rng = np.random.default_rng(0)
    x = np.concatenate([-rng.uniform(0, 125, 1_000_000), -rng.uniform(0, 1, 100_000), np.arange(0, -125, -0.25)])
    x = x.astype(np.float32)
    y = fit.eval_f32(c, x)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 1.2e-4
    # Integer arguments (the largest weight of a row, 2^0, among them) are
    # exact, as on the exponential unit.
    ints = np.arange(0, -126, -1, dtype=np.float32)
    np.testing.assert_array_equal(fit.eval_f32(c, ints), np.exp2(ints))
    # Masked scores and the underflow range give exact zeros.
    assert (fit.eval_f32(c, np.array([-np.inf, -126.0, -200.0], dtype=np.float32)) == 0).all()
    # The largest weight of a row (2^0) still rounds to exactly 1 in bf16.
    one = torch.tensor(fit.eval_f32(c, np.array([0.0], dtype=np.float32))).to(torch.bfloat16)
    assert one.item() == 1.0


@pytest.mark.gpu
def test_device_exp2_poly_against_float64_and_ex2():
    from exact_io_aware_56_b200 import fa

    L = fa.lib()
    L.fa_test_exp2.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_void_p]
    L.fa_test_exp2.restype = ctypes.c_int
    rng = np.random.default_rng(1)
    xs = np.concatenate([-rng.uniform(0, 125, 1 << 20), -rng.uniform(0, 1, 1 << 16), [0.0, -0.5, -125.0],
                         [-np.inf, -126.5, -300.0]]).astype(np.float32)
    x = torch.tensor(xs, device="cuda")
    yp, ye = torch.empty_like(x), torch.empty_like(x)
    assert L.fa_test_exp2(x.data_ptr(), yp.data_ptr(), ye.data_ptr(), x.numel(),
                          torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    torch.cuda.synchronize()
    yp, ye = yp.cpu().numpy().astype(np.float64), ye.cpu().numpy().astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    live = xs >= -125.0
    assert np.max(np.abs(yp[live] / ref[live] - 1.0)) < 1.2e-4
    assert np.max(np.abs(yp[live] / ye[live] - 1.0)) < 1.2e-4 + 1e-6
    assert yp[xs == 0.0][0] == 1.0
    assert (yp[~live] == 0).all()


@pytest.mark.gpu
def test_device_exp2_accurate_against_float64():
    from exact_io_aware_56_b200 import fa

    L = fa.lib()
    L.fa_test_exp2_accurate.argtypes = [ctypes.c_void_p] * 2 + [ctypes.c_int, ctypes.c_void_p]
    L.fa_test_exp2_accurate.restype = ctypes.c_int
    rng = np.random.default_rng(4)
    xs = np.concatenate([-rng.uniform(0, 125, 1 << 20), -rng.uniform(0, 1, 1 << 16), [0.0, -0.5, -125.0],
                         [-np.inf, -126.5, -300.0]]).astype(np.float32)
    x = torch.tensor(xs, device="cuda")
    y = torch.empty_like(x)
    assert L.fa_test_exp2_accurate(x.data_ptr(), y.data_ptr(), x.numel(),
                                   torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    torch.cuda.synchronize()
    y = y.cpu().numpy().astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    live = xs >= -125.0
    assert np.max(np.abs(y[live] / ref[live] - 1.0)) < 5e-7
    assert y[xs == 0.0][0] == 1.0
    assert (y[~live] == 0).all()
