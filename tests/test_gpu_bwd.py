"""GPU parity of the backward kernels against the fp64 oracle (element by
element), on shapes spanning one tile, several tiles, ragged tails and GQA."""

import itertools

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_56_b200 import fa, to_f64

from .parity import assert_close_abs, gpu_inputs, run_fwd

pytestmark = pytest.mark.gpu


def run_bwd(dev, o, lse, causal, scale):
    dq, dk, dv = fa.attention_backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == fa.FA_OK
    return dq, dk, dv


def check_bwd(B, Hq, Hkv, N, d, causal, seed, qk_gain=1.0):
    dev, ref = gpu_inputs(B, Hq, Hkv, N, d, seed, qk_gain)
    scale = d ** -0.5
    o, lse = run_fwd(dev, causal, scale)
    dq, dk, dv = run_bwd(dev, o, lse, causal, scale)
    gq, gk, gv = oracle.attn_bwd_ref(ref["q"], ref["k"], ref["v"], ref["dout"], causal, scale)
    assert_close_abs("dQ", to_f64(dq), gq)
    assert_close_abs("dK", to_f64(dk), gk)
    assert_close_abs("dV", to_f64(dv), gv)


@pytest.mark.parametrize("N,d,causal", list(itertools.product([1, 7, 127, 129, 200, 384], [64, 128],
                                                                [False, True])))
def test_bwd_ragged(N, d, causal):
    check_bwd(2, 2, 2, N, d, causal, seed=N * 3 + d)


@pytest.mark.parametrize("ratio,causal", list(itertools.product([1, 2, 4], [False, True])))
def test_bwd_gqa(ratio, causal):
    check_bwd(1, 4, 4 // ratio, 333, 128, causal, seed=10 + ratio)


@pytest.mark.parametrize("d,causal", list(itertools.product([64, 128], [False, True])))
def test_bwd_many_tiles_peaky(d, causal):
    check_bwd(1, 2, 1, 1100, d, causal, seed=50 + d, qk_gain=2.0)


def test_bwd_workspace_reused_dirty():
    # The workspace may hold garbage from a previous call; results must not depend on it.
    dev, ref = gpu_inputs(1, 2, 2, 300, 64, 77)
    scale = 0.125
    o, lse = run_fwd(dev, True, scale)
    ws = torch.full((fa.fa_bwd_workspace_bytes(1, 2, 2, 300, 64),), 0x7F, dtype=torch.uint8, device="cuda")
    g1 = fa.attention_backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, True, scale, workspace=ws)
    g2 = fa.attention_backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, True, scale, workspace=ws)
    torch.cuda.synchronize()
    gq, gk, gv = oracle.attn_bwd_ref(ref["q"], ref["k"], ref["v"], ref["dout"], True, scale)
    for a, b in zip(g1, g2):
        assert (a.float() - b.float()).abs().max().item() <= 1e-2
    assert_close_abs("dQ", to_f64(g1[0]), gq)
    assert_close_abs("dK", to_f64(g1[1]), gk)
    assert_close_abs("dV", to_f64(g1[2]), gv)


def test_bwd_guard_bytes_untouched():
    B, H, N, d = 1, 2, 260, 128
    dev, ref = gpu_inputs(B, H, H, N, d, 12)
    scale = d ** -0.5
    o, lse = run_fwd(dev, False, scale)
    pad = 8192
    n = B * H * N * d
    bufs = [torch.full((pad + n + pad,), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    dq, dk, dv = (b[pad:pad + n].view(B, H, N, d) for b in bufs)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, H, N, d), dtype=torch.uint8, device="cuda")
    fa.fa_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dq, dk, dv, False, scale, ws)
    torch.cuda.synchronize()
    for b in bufs:
        assert torch.isnan(b[:pad]).all() and torch.isnan(b[-pad:]).all()
    gq, gk, gv = oracle.attn_bwd_ref(ref["q"], ref["k"], ref["v"], ref["dout"], False, scale)
    assert_close_abs("dQ", to_f64(dq), gq)
    assert_close_abs("dK", to_f64(dk), gk)
    assert_close_abs("dV", to_f64(dv), gv)
