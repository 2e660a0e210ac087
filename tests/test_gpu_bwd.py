"""GPU parity of the backward kernels against the fp64 oracle (element by
element), on shapes spanning one tile, several tiles, ragged tails and GQA."""

import itertools

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_56_b200 import fa, to_f64

from .parity import assert_close_abs, assert_close_lse, gpu_inputs, run_bwd, run_fwd

pytestmark = pytest.mark.gpu


def check_bwd(B, Hq, Hkv, N, d, causal, seed, qk_gain=1.0, residual=True):
    """Forward with the O residual, then the backward that uses it (the
    training path), against the exact gradients of the oracle."""
    dev, ref = gpu_inputs(B, Hq, Hkv, N, d, seed, qk_gain)
    scale = d ** -0.5
    if residual:
        o, lse, o_resid = run_fwd(dev, causal, scale, residual=True)
    else:
        (o, lse), o_resid = run_fwd(dev, causal, scale), None
    dq, dk, dv = run_bwd(dev, o, lse, causal, scale, o_resid)
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


@pytest.mark.parametrize("d,causal", list(itertools.product([64, 128], [False, True])))
def test_bwd_plain_entry_point(d, causal):
    # fa_bwd without the residual (D from the bf16 o) on unit-variance inputs.
    check_bwd(2, 4, 2, 500, d, causal, seed=90 + d, residual=False)


def test_fwd_residual_is_rounding_error_of_o():
    dev, ref = gpu_inputs(1, 2, 1, 400, 128, 31, with_dout=False)
    o, lse, r = run_fwd(dev, True, 128 ** -0.5, residual=True)
    # The forward-only call (lazy rescale) and the training call (exact max)
    # agree with the oracle alike; their o may differ in the last bit.
    o2, lse2 = run_fwd(dev, True, 128 ** -0.5)
    O, L = oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], True, 128 ** -0.5)
    for oo, ll in ((o, lse), (o2, lse2)):
        assert_close_abs("O", to_f64(oo), O)
        assert_close_lse(to_f64(ll), L)
    hi, lo = to_f64(o), to_f64(r)
    # o_resid is a rounding residual of o: at most half an ulp of o (bf16 has
    # 8 significant bits, so half an ulp is 2^-8 * 2^floor(log2|o|)).
    half_ulp = np.where(hi != 0, 2.0 ** (np.floor(np.log2(np.abs(np.where(hi != 0, hi, 1.0)))) - 8), 2.0 ** -133)
    assert (np.abs(lo) <= half_ulp).all()
    # and o + o_resid is on average closer to the exact O than o alone.
    assert np.abs(hi + lo - O).mean() < 0.75 * np.abs(hi - O).mean()


def test_bwd_workspace_reused_dirty():
    # The workspace may hold garbage from a previous call; results must not depend on it.
    dev, ref = gpu_inputs(1, 2, 2, 300, 64, 77)
    scale = 0.125
    o, lse, r = run_fwd(dev, True, scale, residual=True)
    ws = torch.full((fa.fa_bwd_workspace_bytes(1, 2, 2, 300, 64),), 0x7F, dtype=torch.uint8, device="cuda")
    g1 = fa.attention_backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, True, scale, workspace=ws,
                               o_resid=r)
    g2 = fa.attention_backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, True, scale, workspace=ws,
                               o_resid=r)
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
    o, lse, r = run_fwd(dev, False, scale, residual=True)
    pad = 8192
    n = B * H * N * d
    bufs = [torch.full((pad + n + pad,), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    dq, dk, dv = (b[pad:pad + n].view(B, H, N, d) for b in bufs)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, H, N, d), dtype=torch.uint8, device="cuda")
    fa.fa_bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, dq, dk, dv, False, scale, ws, o_resid=r)
    torch.cuda.synchronize()
    for b in bufs:
        assert torch.isnan(b[:pad]).all() and torch.isnan(b[-pad:]).all()
    gq, gk, gv = oracle.attn_bwd_ref(ref["q"], ref["k"], ref["v"], ref["dout"], False, scale)
    assert_close_abs("dQ", to_f64(dq), gq)
    assert_close_abs("dK", to_f64(dk), gk)
    assert_close_abs("dV", to_f64(dv), gv)
