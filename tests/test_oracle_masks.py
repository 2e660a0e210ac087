"""Pins of the oracle's sliding-window and prefix-LM masks: reductions to the
causal and full masks, closed forms, pure-Python brute force, online ==
two-pass, and finite differences of the backward."""

import itertools
import math

import numpy as np
import pytest

import oracle
from oracle import attention as A

from .test_oracle_pins import brute_fwd, loss, rnd


def brute_fwd_masked(q, k, v, scale, window, prefix):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    O = np.zeros(q.shape)
    L = np.zeros((B, Hq, N))
    for b, h, i in itertools.product(range(B), range(Hq), range(N)):
        g = h // (Hq // Hkv)
        vis = [j for j in range(N) if (j <= i and (window is None or i - j <= window)) or j < prefix]
        s = [scale * math.fsum(q[b, h, i, c] * k[b, g, j, c] for c in range(d)) for j in vis]
        e = [math.exp(x) for x in s]
        tot = math.fsum(e)
        L[b, h, i] = math.log(tot)
        for c in range(d):
            O[b, h, i, c] = math.fsum(e[t] * v[b, g, j, c] for t, j in enumerate(vis)) / tot
    return O, L


CASES = [(None, 0), (0, 0), (1, 0), (3, 0), (None, 2), (None, 5), (2, 3), (0, 4)]


@pytest.mark.parametrize("window,prefix", CASES)
def test_masked_brute_force(window, prefix):
    q, k, v = rnd((1, 2, 7, 3), 201), rnd((1, 1, 7, 3), 202), rnd((1, 1, 7, 3), 203)
    O, L = oracle.attn_fwd_ref(q, k, v, True, 0.8, window, prefix)
    Ob, Lb = brute_fwd_masked(q, k, v, 0.8, window, prefix)
    np.testing.assert_allclose(O, Ob, atol=1e-13)
    np.testing.assert_allclose(L, Lb, atol=1e-13)


def test_mask_reductions():
    q, k, v = rnd((2, 2, 40, 5), 211, 2.0), rnd((2, 2, 40, 5), 212, 2.0), rnd((2, 2, 40, 5), 213)
    causal = oracle.attn_fwd_ref(q, k, v, True, 0.5)
    full = oracle.attn_fwd_ref(q, k, v, False, 0.5)
    for window in (39, 100):   # a window covering every earlier key is plain causal
        got = oracle.attn_fwd_ref(q, k, v, True, 0.5, window, 0)
        np.testing.assert_allclose(got[0], causal[0], atol=0)
    got = oracle.attn_fwd_ref(q, k, v, True, 0.5, None, 40)  # a prefix of all keys is full attention
    np.testing.assert_allclose(got[0], full[0], atol=1e-14)
    np.testing.assert_allclose(got[1], full[1], atol=1e-14)
    got = oracle.attn_fwd_ref(q, k, v, True, 0.5, None, 1)   # a prefix of one key adds nothing
    np.testing.assert_allclose(got[0], causal[0], atol=0)


def test_window_zero_returns_own_value_row():
    q, k, v = rnd((1, 3, 25, 4), 221), rnd((1, 3, 25, 4), 222), rnd((1, 3, 25, 4), 223)
    O, L = oracle.attn_fwd_ref(q, k, v, True, 0.7, 0, 0)
    np.testing.assert_allclose(O, v, atol=1e-15)
    np.testing.assert_allclose(L, 0.7 * (q * k).sum(-1), atol=1e-14)


@pytest.mark.parametrize("window,prefix", [(4, 0), (None, 6), (3, 5)])
def test_zero_q_mean_of_visible_rows(window, prefix):
    N = 20
    v = rnd((1, 1, N, 3), 231)
    q = np.zeros((1, 1, N, 3))
    k = rnd((1, 1, N, 3), 232)
    O, L = oracle.attn_fwd_ref(q, k, v, True, 1.0, window, prefix)
    vis = A.visible(np.arange(N), np.arange(N), True, window, prefix)
    cnt = vis.sum(1)
    np.testing.assert_allclose(O[0, 0], (vis @ v[0, 0]) / cnt[:, None], atol=1e-14)
    np.testing.assert_allclose(L[0, 0], np.log(cnt), atol=1e-14)


@pytest.mark.parametrize("window,prefix", [(5, 0), (None, 9), (4, 7)])
def test_masked_online_equals_two_pass(window, prefix):
    q, k, v = rnd((1, 2, 50, 6), 241, 2.0), rnd((1, 1, 50, 6), 242, 2.0), rnd((1, 1, 50, 6), 243)
    O, L = oracle.attn_fwd_ref(q, k, v, True, 0.5, window, prefix)
    for bq, bk in [(1, 1), (7, 5), (16, 16), (50, 50)]:
        Oo, Lo = oracle.attn_fwd_online_ref(q, k, v, True, 0.5, bq, bk, window, prefix)
        np.testing.assert_allclose(Oo, O, atol=1e-12)
        np.testing.assert_allclose(Lo, L, atol=1e-12)


@pytest.mark.parametrize("window,prefix", [(1, 0), (None, 3), (2, 2)])
def test_masked_backward_finite_differences(window, prefix):
    h = 1e-6
    q, k, v, do = rnd((1, 2, 6, 3), 251), rnd((1, 1, 6, 3), 252), rnd((1, 1, 6, 3), 253), rnd((1, 2, 6, 3), 254)
    fwd = lambda q_, k_, v_, c, s: oracle.attn_fwd_ref(q_, k_, v_, c, s, window, prefix)
    grads = oracle.attn_bwd_ref(q, k, v, do, True, 0.9, window, prefix)
    for which, g in zip("qkv", grads):
        arrs = {"q": q, "k": k, "v": v}
        x = arrs[which]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            ap, am = dict(arrs, **{which: xp}), dict(arrs, **{which: xm})
            fd[idx] = (loss(ap["q"], ap["k"], ap["v"], do, True, 0.9, fwd)
                       - loss(am["q"], am["k"], am["v"], do, True, 0.9, fwd)) / (2 * h)
        assert np.abs(fd - g).max() / max(1.0, np.abs(fd).max()) < 1e-6, which


def test_masked_sampled_variants_equal_full():
    q, k, v, do = rnd((1, 4, 60, 5), 261), rnd((1, 2, 60, 5), 262), rnd((1, 2, 60, 5), 263), rnd((1, 4, 60, 5), 264)
    rows = np.array([0, 3, 17, 40, 59])
    for window, prefix in [(7, 0), (None, 11), (5, 9)]:
        O, L = oracle.attn_fwd_ref(q, k, v, True, 0.4, window, prefix)
        dq, dk, dv = oracle.attn_bwd_ref(q, k, v, do, True, 0.4, window, prefix)
        Or, Lr = oracle.attn_fwd_rows(q, k, v, True, 0.4, 0, 3, rows, window, prefix)
        np.testing.assert_allclose(Or, O[0, 3, rows], atol=1e-14)
        np.testing.assert_allclose(Lr, L[0, 3, rows], atol=1e-14)
        np.testing.assert_allclose(oracle.attn_bwd_rows(q, k, v, do, True, 0.4, 0, 2, rows, window, prefix),
                                   dq[0, 2, rows], atol=1e-13)
        dkr, dvr = oracle.attn_bwd_kv_rows(q, k, v, do, True, 0.4, 0, 1, rows, window, prefix)
        np.testing.assert_allclose(dkr, dk[0, 1, rows], atol=1e-13)
        np.testing.assert_allclose(dvr, dv[0, 1, rows], atol=1e-13)


def _check_masked_brute():
    for window, prefix in CASES:
        q, k, v = rnd((1, 2, 7, 3), 201), rnd((1, 1, 7, 3), 202), rnd((1, 1, 7, 3), 203)
        O, L = oracle.attn_fwd_ref(q, k, v, True, 0.8, window, prefix)
        Ob, Lb = brute_fwd_masked(q, k, v, 0.8, window, prefix)
        np.testing.assert_allclose(O, Ob, atol=1e-13)


_orig_visible = A.visible


@pytest.mark.parametrize("kind", ["window off by one", "prefix off by one"])
def test_mask_mutation_is_caught(monkeypatch, kind):
    def bad(row_ids, col_ids, causal, window=None, prefix=0):
        if kind == "window off by one" and window is not None:
            window = window + 1
        if kind == "prefix off by one" and prefix:
            prefix = prefix + 1
        return _orig_visible(row_ids, col_ids, causal, window, prefix)

    monkeypatch.setattr(A, "visible", bad)
    with pytest.raises(AssertionError):
        _check_masked_brute()
