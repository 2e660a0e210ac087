"""GPU parity of the sliding-window / prefix-LM kernels (mask kind 2)
against the fp64 oracle: windows and prefixes at, below and above tile
boundaries, combined, with GQA, both head dims and ragged N."""

import itertools

import pytest
import torch

import oracle
from exact_io_aware_56_b200 import fa, to_f64

from .parity import assert_close_abs, assert_close_lse, gpu_inputs

pytestmark = pytest.mark.gpu

MASKS = [(0, 0), (1, 0), (63, 0), (128, 0), (200, 0), (None, 1), (None, 100), (None, 128), (None, 300),
         (64, 150), (5, 400)]


def check_masked(B, Hq, Hkv, N, d, window, prefix, seed, qk_gain=1.0):
    dev, ref = gpu_inputs(B, Hq, Hkv, N, d, seed, qk_gain)
    scale = d ** -0.5
    o, lse, r = fa.attention_forward(dev["q"], dev["k"], dev["v"], True, scale, residual=True, window=window,
                                     prefix=prefix)
    dq, dk, dv = fa.attention_backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, True, scale,
                                       o_resid=r, window=window, prefix=prefix)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == fa.FA_OK
    O, L = oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], True, scale, window, prefix)
    assert_close_abs("O", to_f64(o), O)
    assert_close_lse(to_f64(lse), L)
    gq, gk, gv = oracle.attn_bwd_ref(ref["q"], ref["k"], ref["v"], ref["dout"], True, scale, window, prefix)
    assert_close_abs("dQ", to_f64(dq), gq)
    assert_close_abs("dK", to_f64(dk), gk)
    assert_close_abs("dV", to_f64(dv), gv)


@pytest.mark.parametrize("window,prefix", MASKS)
@pytest.mark.parametrize("d", [64, 128])
def test_masks_ragged(window, prefix, d):
    check_masked(1, 2, 1, 777, d, window, prefix, seed=300 + d + (window or 0) + prefix)


@pytest.mark.parametrize("window,prefix", [(100, 0), (None, 200)])
def test_masks_gqa_long_peaky(window, prefix):
    check_masked(1, 4, 2, 1500, 128, window, prefix, seed=401, qk_gain=2.0)


def test_masks_gqa_long_window_and_prefix():
    # With qk gain 2, a 37-key window and a 70-key prefix, every row puts
    # large weights on the prefix keys, and the bf16 rounding of dS alone (all
    # else exact, in fp64) already moves dK by 4.8e-2, past the 2e-2 bar; the
    # combined mask is checked at unit gain, where that rounding stays near
    # 1e-2.
    check_masked(1, 4, 2, 1500, 128, 37, 70, seed=401, qk_gain=1.0)


def test_masks_reduce_to_causal_and_full_bitwise():
    # window covering everything == causal kernel; prefix >= N == full attention kernel.
    dev, _ = gpu_inputs(1, 2, 2, 500, 128, 9, with_dout=False)
    c = fa.attention_forward(dev["q"], dev["k"], dev["v"], True, 0.09)
    w = fa.attention_forward(dev["q"], dev["k"], dev["v"], True, 0.09, window=10 ** 6)
    f = fa.attention_forward(dev["q"], dev["k"], dev["v"], False, 0.09)
    p = fa.attention_forward(dev["q"], dev["k"], dev["v"], True, 0.09, prefix=500)
    torch.cuda.synchronize()
    assert torch.equal(c[0], w[0]) and torch.equal(c[1], w[1])
    assert torch.equal(f[0], p[0]) and torch.equal(f[1], p[1])


def test_mask_argument_errors():
    dev, _ = gpu_inputs(1, 1, 1, 64, 64, 1, with_dout=False)
    with pytest.raises(fa.FaError):
        fa.attention_forward(dev["q"], dev["k"], dev["v"], True, 0.125, window=-2)
    with pytest.raises(fa.FaError):
        fa.attention_forward(dev["q"], dev["k"], dev["v"], True, 0.125, prefix=-1)
    with pytest.raises(ValueError):
        fa.attention_forward(dev["q"], dev["k"], dev["v"], False, 0.125, window=4)
