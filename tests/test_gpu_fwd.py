"""GPU parity of the forward kernel against the fp64 oracle (element by
element), on shapes spanning one tile, several tiles and ragged tails."""

import itertools

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_56_b200 import WORKLOADS, fa, to_f64

from .parity import assert_close_abs, assert_close_lse, gpu_inputs, run_fwd

pytestmark = pytest.mark.gpu


def check_fwd(B, Hq, Hkv, N, d, causal, seed, qk_gain=1.0):
    dev, ref = gpu_inputs(B, Hq, Hkv, N, d, seed, qk_gain, with_dout=False)
    scale = d ** -0.5
    o, lse = run_fwd(dev, causal, scale)
    O, L = oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], causal, scale)
    assert_close_abs("O", to_f64(o), O)
    assert_close_lse(to_f64(lse), L)


def test_fwd_single_tile_n128_d64():
    w = WORKLOADS["fwd_b1_h1_n128_d64"]
    check_fwd(w.B, w.Hq, w.Hkv, w.N, w.d, w.causal, w.seed)


@pytest.mark.parametrize("N,d,causal", list(itertools.product([1, 7, 127, 129, 200, 384], [64, 128],
                                                                [False, True])))
def test_fwd_ragged(N, d, causal):
    check_fwd(2, 2, 2, N, d, causal, seed=N * 7 + d)


@pytest.mark.parametrize("ratio,causal", list(itertools.product([1, 2, 4], [False, True])))
def test_fwd_gqa(ratio, causal):
    check_fwd(1, 4, 4 // ratio, 333, 128, causal, seed=ratio)


@pytest.mark.parametrize("d,causal", list(itertools.product([64, 128], [False, True])))
def test_fwd_many_tiles_peaky(d, causal):
    # Large scores stress the running-max rescale.
    check_fwd(1, 2, 1, 1100, d, causal, seed=5 + d, qk_gain=2.0)


def rising_inputs(B, H, N, d, seed, step_log2=3.0):
    """Q, K, V (bf16, CPU) whose scores grow along the key axis: every query
    gets a shared unit direction u with weight 4 and key j gets u with weight
    beta * j, so each 128-key tile raises a row's max by about `step_log2`
    (log2 units) on top of unit-variance noise."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    u = torch.randn(d, generator=g, dtype=torch.float64)
    u /= u.norm()
    beta = step_log2 / (4.0 * 128 * d ** -0.5 * np.log2(np.e))
    q += 4.0 * u
    k += beta * torch.arange(N, dtype=torch.float64).view(1, 1, N, 1) * u
    return {"q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16), "v": v.to(torch.bfloat16)}


@pytest.mark.parametrize("d,causal", list(itertools.product([64, 128], [False, True])))
def test_fwd_rising_scores_deferred_and_exact_rescale(d, causal):
    # Row maxima that keep growing across tiles: the forward-only call defers
    # the O rescale until a max grew by more than 8 (log2), so P carries
    # weights up to 2^8 between rescales; the training call rescales at every
    # growth. Both must match the oracle.
    B, H, N = 1, 2, 1100
    host = rising_inputs(B, H, N, d, seed=90 + d)
    ref = {n: to_f64(t) for n, t in host.items()}
    scale = d ** -0.5
    # The inputs do what the test needs: per-tile maxima of a row rise by
    # less than 8 from one tile to the next but by far more over the row.
    S = scale * np.log2(np.e) * ref["q"][0, 0, -1] @ ref["k"][0, 0].T
    tile_max = np.maximum.accumulate([S[t:t + 128].max() for t in range(0, N, 128)])
    steps = np.diff(tile_max)
    assert (steps < 8).all() and tile_max[-1] - tile_max[0] > 16
    dev = {n: t.cuda() for n, t in host.items()}
    O, L = oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], causal, scale)
    o, lse = run_fwd(dev, causal, scale)
    assert_close_abs("O lazy", to_f64(o), O)
    assert_close_lse(to_f64(lse), L)
    o, lse, _ = run_fwd(dev, causal, scale, residual=True)
    assert_close_abs("O exact", to_f64(o), O)
    assert_close_lse(to_f64(lse), L)


def test_fwd_deterministic():
    dev, _ = gpu_inputs(1, 2, 2, 700, 128, 3, with_dout=False)
    o1, l1 = run_fwd(dev, True, 128 ** -0.5)
    o2, l2 = run_fwd(dev, True, 128 ** -0.5)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_guard_bytes_untouched():
    # Outputs sit inside larger buffers filled with a sentinel; the bytes
    # around them must be unchanged after the call.
    B, H, N, d = 1, 3, 300, 64
    dev, ref = gpu_inputs(B, H, H, N, d, 11, with_dout=False)
    pad = 16384
    ob = torch.full((pad + B * H * N * d + pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
    lb = torch.full((pad + B * H * N + pad,), 12345.0, dtype=torch.float32, device="cuda")
    o = ob[pad:pad + B * H * N * d].view(B, H, N, d)
    lse = lb[pad:pad + B * H * N].view(B, H, N)
    fa.fa_fwd(dev["q"], dev["k"], dev["v"], o, lse, True, d ** -0.5)
    torch.cuda.synchronize()
    assert torch.isnan(ob[:pad]).all() and torch.isnan(ob[-pad:]).all()
    assert (lb[:pad] == 12345.0).all() and (lb[-pad:] == 12345.0).all()
    O, L = oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], True, d ** -0.5)
    assert_close_abs("O", to_f64(o), O)
    assert_close_lse(to_f64(lse), L)
