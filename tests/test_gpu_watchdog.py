"""Failure detection without a GPU fault: the test hook makes the forward
producer skip one K tile, so the MMA thread's wait can never be satisfied.
The bounded wait must run out, the CTA must drain and exit, the host must
read FA_ERR_TIMEOUT, and the context must stay usable."""

import pytest
import torch

import oracle
from exact_io_aware_56_b200 import fa, to_f64

from .parity import assert_close_abs, assert_close_lse, gpu_inputs, run_fwd

pytestmark = pytest.mark.gpu


def test_forward_wait_times_out_cleanly_and_context_recovers():
    dev, ref = gpu_inputs(1, 2, 2, 300, 64, seed=21, with_dout=False)
    o = torch.empty_like(dev["q"])
    lse = torch.empty((1, 2, 300), dtype=torch.float32, device="cuda")
    assert fa.fa_check_device_error() == fa.FA_OK
    fa.fa_set_watchdog_ns(50_000_000)
    fa.fa_test_set_fault(1)
    try:
        fa.fa_fwd(dev["q"], dev["k"], dev["v"], o, lse, False, 0.125)
        assert fa.fa_check_device_error() == fa.FA_ERR_TIMEOUT
        # The word was cleared by the read.
        assert fa.fa_check_device_error() == fa.FA_OK
    finally:
        fa.fa_test_set_fault(0)
        fa.fa_set_watchdog_ns(2_000_000_000)
    out, l2 = run_fwd(dev, False, 0.125)
    O, L = oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], False, 0.125)
    assert_close_abs("O", to_f64(out), O)
    assert_close_lse(to_f64(l2), L)
