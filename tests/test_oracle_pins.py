"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each check ties the oracle to something fixed independently of its own code:
a closed form, an identity of the definition, pure-Python brute force on tiny
inputs, central finite differences, or a second library (torch autograd in
fp64 on the CPU). ``test_oracle_mutations.py`` plants mistakes in the oracle
and shows that these checks catch them.
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- brute force

def brute_fwd(q, k, v, causal, scale):
    """Pure-Python loops: S_ij, exp, math.fsum for the sums. Tiny sizes only."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    O = np.zeros(q.shape)
    L = np.zeros((B, Hq, N))
    for b, h, i in itertools.product(range(B), range(Hq), range(N)):
        g = h // (Hq // Hkv)
        vis = [j for j in range(N) if not (causal and j > i)]
        s = [scale * math.fsum(q[b, h, i, c] * k[b, g, j, c] for c in range(d)) for j in vis]
        e = [math.exp(x) for x in s]
        tot = math.fsum(e)
        L[b, h, i] = math.log(tot)
        for c in range(d):
            O[b, h, i, c] = math.fsum(e[t] * v[b, g, j, c] for t, j in enumerate(vis)) / tot
    return O, L


def check_brute_force(fwd=None):
    fwd = fwd or oracle.attn_fwd_ref
    for causal, (Hq, Hkv), N in itertools.product([False, True], [(1, 1), (2, 1), (4, 2)], [1, 3, 5]):
        d = 3
        q = rnd((2, Hq, N, d), 1 + N)
        k = rnd((2, Hkv, N, d), 2 + N)
        v = rnd((2, Hkv, N, d), 3 + N)
        O, L = fwd(q, k, v, causal, 0.7)
        Ob, Lb = brute_fwd(q, k, v, causal, 0.7)
        np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-13)
        np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-13)


def test_brute_force_tiny():
    check_brute_force()


def test_closed_form_two_keys():
    # q = e0, keys e0 and e1, scale 1: scores (1, 0), so p = (e, 1) / (e + 1).
    q = np.array([1.0, 0.0]).reshape(1, 1, 1, 2)
    k = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 1, 2, 2)
    v = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(1, 1, 2, 2)
    # Two rows for k/v but one query row: pad q to N = 2 with a second row.
    q = np.concatenate([q, np.zeros((1, 1, 1, 2))], axis=2)
    O, L = oracle.attn_fwd_ref(q, k, v, False, 1.0)
    p0 = math.e / (math.e + 1.0)
    np.testing.assert_allclose(O[0, 0, 0], [p0 * 1 + (1 - p0) * 3, p0 * 2 + (1 - p0) * 4], atol=1e-15)
    assert abs(L[0, 0, 0] - math.log(math.e + 1.0)) < 1e-15
    # Second query is zero: uniform weights, L = ln 2.
    np.testing.assert_allclose(O[0, 0, 1], [2.0, 3.0], atol=1e-15)
    assert abs(L[0, 0, 1] - math.log(2.0)) < 1e-15


# --------------------------------------------------------------- identities

def check_online_equals_two_pass(online=None, ref=None):
    online = online or oracle.attn_fwd_online_ref
    ref = ref or oracle.attn_fwd_ref
    rng = np.random.default_rng(7)
    for causal, (Hq, Hkv), N in itertools.product([False, True], [(2, 2), (4, 1)], [1, 17, 64, 100]):
        d = 8
        q = rnd((1, Hq, N, d), 11 + N, 2.0)
        k = rnd((1, Hkv, N, d), 12 + N, 2.0)
        v = rnd((1, Hkv, N, d), 13 + N)
        O, L = ref(q, k, v, causal, 0.5)
        for bq, bk in [(1, 1), (N, N), (128, 128)] + [tuple(rng.integers(1, N + 1, 2)) for _ in range(2)]:
            Oo, Lo = online(q, k, v, causal, 0.5, int(bq), int(bk))
            np.testing.assert_allclose(Oo, O, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(Lo, L, rtol=1e-12, atol=1e-12)


def test_online_equals_two_pass():
    check_online_equals_two_pass()


def check_online_any_merge_order():
    # The merge of partial softmax states is associative and commutative, so
    # merging the key blocks in any order gives the two-pass result.
    rng = np.random.default_rng(71)
    for causal, N, bk in [(False, 37, 5), (True, 37, 5), (True, 64, 16), (False, 9, 1)]:
        q = rnd((1, 2, N, 6), 71 + N, 2.0)
        k = rnd((1, 1, N, 6), 72 + N, 2.0)
        v = rnd((1, 1, N, 6), 73 + N)
        O, L = oracle.attn_fwd_ref(q, k, v, causal, 0.7)
        nb = (N + bk - 1) // bk
        for order in [list(range(nb))[::-1], list(rng.permutation(nb)), list(rng.permutation(nb))]:
            Oo, Lo = oracle.attn_fwd_online_ref(q, k, v, causal, 0.7, 7, bk, order=order)
            np.testing.assert_allclose(Oo, O, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(Lo, L, rtol=1e-12, atol=1e-12)


def test_online_any_merge_order():
    check_online_any_merge_order()


def check_merge_closed_form():
    # Two keys with scores s1, s2 and values v1, v2, one per block: the merged
    # state must give softmax weights e^s / (e^s1 + e^s2) and L = ln(e^s1 + e^s2),
    # computed here with math.exp / math.fsum.
    for s1, s2 in [(0.3, -1.2), (5.0, 5.0), (-40.0, 2.5), (700.0, 699.0)]:
        v1, v2 = np.array([1.0, -2.0, 0.5]), np.array([3.0, 0.25, -1.0])
        a = oracle.softmax_state(np.array([[s1]]), v1[None])
        b = oracle.softmax_state(np.array([[s2]]), v2[None])
        mx = max(s1, s2)
        e1, e2 = math.exp(s1 - mx), math.exp(s2 - mx)
        want_o = (e1 * v1 + e2 * v2) / math.fsum([e1, e2])
        want_l = mx + math.log(math.fsum([e1, e2]))
        for m, l, U in (oracle.merge_softmax_states(a, b), oracle.merge_softmax_states(b, a)):
            np.testing.assert_allclose(U[0] / l[0], want_o, rtol=1e-14, atol=1e-14)
            assert abs(m[0] + math.log(l[0]) - want_l) <= 1e-12 * max(1.0, abs(want_l))
    # The empty state (every key of a block masked) is the identity, exactly.
    empty = oracle.softmax_state(np.full((1, 4), -np.inf), np.ones((4, 3)))
    assert np.isneginf(empty[0]).all() and (empty[1] == 0).all() and (empty[2] == 0).all()
    a = oracle.softmax_state(np.array([[0.5, -0.25]]), np.array([[1.0, 2.0, 3.0], [4.0, 5.0, 6.0]]))
    for merged in (oracle.merge_softmax_states(a, empty), oracle.merge_softmax_states(empty, a)):
        for x, y in zip(merged, a):
            assert np.array_equal(x, y)


def test_merge_closed_form():
    check_merge_closed_form()


def test_online_matches_brute_force():
    # The blocked online form against pure-Python loops (independent of the
    # two-pass oracle), causal and not, blocks that do not divide N.
    for causal in (False, True):
        q = rnd((1, 2, 7, 3), 91, 1.5)
        k = rnd((1, 1, 7, 3), 92, 1.5)
        v = rnd((1, 1, 7, 3), 93)
        O, L = brute_fwd(q, k, v, causal, 0.8)
        Oo, Lo = oracle.attn_fwd_online_ref(q, k, v, causal, 0.8, 3, 2)
        np.testing.assert_allclose(Oo, O, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(Lo, L, rtol=1e-13, atol=1e-13)


def check_rows_sum_to_one(fwd=None):
    # A V column of ones returns sum_j P_ij, which must be 1 in every row.
    fwd = fwd or oracle.attn_fwd_ref
    for causal in (False, True):
        q = rnd((2, 2, 33, 6), 21, 3.0)
        k = rnd((2, 2, 33, 6), 22, 3.0)
        v = rnd((2, 2, 33, 6), 23)
        v[..., 0] = 1.0
        O, _ = fwd(q, k, v, causal, 0.4)
        np.testing.assert_allclose(O[..., 0], 1.0, rtol=0, atol=1e-14)


def test_rows_of_p_sum_to_one():
    check_rows_sum_to_one()


def check_constant_v(fwd=None):
    fwd = fwd or oracle.attn_fwd_ref
    c = np.array([0.5, -2.0, 3.25, 1.0])
    for causal in (False, True):
        q = rnd((1, 2, 40, 4), 31, 2.0)
        k = rnd((1, 1, 40, 4), 32, 2.0)
        v = np.broadcast_to(c, (1, 1, 40, 4)).copy()
        O, _ = fwd(q, k, v, causal, 0.3)
        np.testing.assert_allclose(O, np.broadcast_to(c, O.shape), rtol=0, atol=1e-14)


def test_constant_v_returns_constant():
    check_constant_v()


def check_zero_q(fwd=None):
    fwd = fwd or oracle.attn_fwd_ref
    N, d = 37, 5
    v = rnd((1, 2, N, d), 41)
    k = rnd((1, 2, N, d), 42)
    q = np.zeros((1, 2, N, d))
    O, L = fwd(q, k, v, False, 0.9)
    np.testing.assert_allclose(O, np.broadcast_to(v.mean(axis=2, keepdims=True), O.shape), atol=1e-14)
    np.testing.assert_allclose(L, math.log(N), atol=1e-14)
    O, L = fwd(q, k, v, True, 0.9)
    prefix = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    np.testing.assert_allclose(O, prefix, atol=1e-14)
    np.testing.assert_allclose(L, np.log(np.arange(1, N + 1))[None, None, :].repeat(2, 1), atol=1e-14)


def test_zero_q_returns_mean_of_visible_v():
    check_zero_q()


def check_causal_row0(fwd=None):
    fwd = fwd or oracle.attn_fwd_ref
    q = rnd((2, 3, 9, 4), 51)
    k = rnd((2, 3, 9, 4), 52)
    v = rnd((2, 3, 9, 4), 53)
    O, L = fwd(q, k, v, True, 0.6)
    np.testing.assert_allclose(O[:, :, 0], v[:, :, 0], atol=1e-15)
    np.testing.assert_allclose(L[:, :, 0], 0.6 * (q[:, :, 0] * k[:, :, 0]).sum(-1), atol=1e-14)


def test_causal_row0():
    check_causal_row0()


def check_permutation_invariance(fwd=None):
    fwd = fwd or oracle.attn_fwd_ref
    q = rnd((1, 2, 20, 4), 61, 2.0)
    k = rnd((1, 2, 20, 4), 62, 2.0)
    v = rnd((1, 2, 20, 4), 63)
    perm = np.random.default_rng(64).permutation(20)
    O, L = fwd(q, k, v, False, 0.5)
    Op, Lp = fwd(q, k[:, :, perm], v[:, :, perm], False, 0.5)
    np.testing.assert_allclose(Op, O, atol=1e-13)
    np.testing.assert_allclose(Lp, L, atol=1e-13)
    Oq, Lq = fwd(q[:, :, perm], k, v, False, 0.5)
    np.testing.assert_allclose(Oq, O[:, :, perm], atol=1e-13)
    np.testing.assert_allclose(Lq, L[:, :, perm], atol=1e-13)


def test_permutation_invariance():
    check_permutation_invariance()


def test_gqa_equals_repeated_kv():
    # Query head h with KV head h // r equals plain MHA on repeated K, V.
    q = rnd((2, 6, 11, 4), 71)
    k = rnd((2, 2, 11, 4), 72)
    v = rnd((2, 2, 11, 4), 73)
    for causal in (False, True):
        O, L = oracle.attn_fwd_ref(q, k, v, causal, 0.5)
        Om, Lm = oracle.attn_fwd_ref(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), causal, 0.5)
        np.testing.assert_allclose(O, Om, atol=0)
        np.testing.assert_allclose(L, Lm, atol=0)
    assert [oracle.kv_head_of(h, 6, 2) for h in range(6)] == [0, 0, 0, 1, 1, 1]


def test_no_overflow_on_large_scores():
    # Scores around 1e3 overflow a plain exp; the max-shifted forms must not.
    q = rnd((1, 1, 16, 4), 81, 30.0)
    k = rnd((1, 1, 16, 4), 82, 30.0)
    v = rnd((1, 1, 16, 4), 83)
    O, L = oracle.attn_fwd_ref(q, k, v, True, 1.0)
    Oo, Lo = oracle.attn_fwd_online_ref(q, k, v, True, 1.0, 4, 3)
    assert np.isfinite(O).all() and np.isfinite(L).all()
    np.testing.assert_allclose(Oo, O, atol=1e-12)
    np.testing.assert_allclose(Lo, L, rtol=1e-14)


# ------------------------------------------------------------------ backward

def loss(q, k, v, dout, causal, scale, fwd=None):
    fwd = fwd or oracle.attn_fwd_ref
    O, _ = fwd(q, k, v, causal, scale)
    return float((O * dout).sum())


def check_backward_fd(bwd=None):
    bwd = bwd or oracle.attn_bwd_ref
    h = 1e-6
    for causal, (Hq, Hkv), N, d in [(False, (1, 1), 5, 3), (True, (2, 2), 6, 4), (True, (2, 1), 7, 3),
                                    (False, (4, 2), 4, 2)]:
        q = rnd((1, Hq, N, d), 91 + N)
        k = rnd((1, Hkv, N, d), 92 + N)
        v = rnd((1, Hkv, N, d), 93 + N)
        dout = rnd((1, Hq, N, d), 94 + N)
        grads = bwd(q, k, v, dout, causal, 0.8)
        for which, g in zip("qkv", grads):
            arrs = {"q": q, "k": k, "v": v}
            x = arrs[which]
            fd = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp = x.copy(); xp[idx] += h
                xm = x.copy(); xm[idx] -= h
                ap = dict(arrs); ap[which] = xp
                am = dict(arrs); am[which] = xm
                fd[idx] = (loss(ap["q"], ap["k"], ap["v"], dout, causal, 0.8)
                           - loss(am["q"], am["k"], am["v"], dout, causal, 0.8)) / (2 * h)
            err = np.abs(fd - g).max() / max(1.0, np.abs(fd).max())
            assert err < 1e-6, (which, causal, Hq, Hkv, err)


def test_backward_matches_finite_differences():
    check_backward_fd()


def test_backward_d_identity():
    # D_i = sum_j P_ij dP_ij equals sum_c dO_ic O_ic (used by the kernels' preprocess).
    q = rnd((1, 2, 30, 5), 101, 2.0)
    k = rnd((1, 2, 30, 5), 102, 2.0)
    v = rnd((1, 2, 30, 5), 103)
    dout = rnd((1, 2, 30, 5), 104)
    for causal in (False, True):
        O, L = oracle.attn_fwd_ref(q, k, v, causal, 0.5)
        for h in range(2):
            S = 0.5 * q[0, h] @ k[0, h].T
            if causal:
                S[np.triu_indices(30, 1)] = -np.inf
            P = np.exp(S - L[0, h][:, None])
            dP = dout[0, h] @ v[0, h].T
            np.testing.assert_allclose((P * dP).sum(1), (dout[0, h] * O[0, h]).sum(1), atol=1e-12)


def test_backward_matches_torch_autograd_fp64():
    q = rnd((2, 4, 19, 6), 111)
    k = rnd((2, 2, 19, 6), 112)
    v = rnd((2, 2, 19, 6), 113)
    dout = rnd((2, 4, 19, 6), 114)
    for causal in (False, True):
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        S = 0.45 * tq @ tk.repeat_interleave(2, dim=1).transpose(-1, -2)
        if causal:
            S = S.masked_fill(torch.ones(19, 19, dtype=torch.bool).triu(1), float("-inf"))
        O = torch.softmax(S, dim=-1) @ tv.repeat_interleave(2, dim=1)
        (O * torch.tensor(dout)).sum().backward()
        dq, dk, dv = oracle.attn_bwd_ref(q, k, v, dout, causal, 0.45)
        np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
        np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
        np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12)
        Oo, _ = oracle.attn_fwd_ref(q, k, v, causal, 0.45)
        np.testing.assert_allclose(Oo, O.detach().numpy(), atol=1e-13)


# ----------------------------------------------------------- sampled variants

def test_sampled_rows_equal_full():
    q = rnd((2, 4, 70, 8), 121, 2.0)
    k = rnd((2, 2, 70, 8), 122, 2.0)
    v = rnd((2, 2, 70, 8), 123)
    dout = rnd((2, 4, 70, 8), 124)
    rows = np.array([0, 5, 33, 69])
    for causal in (False, True):
        O, L = oracle.attn_fwd_ref(q, k, v, causal, 0.35)
        dq, dk, dv = oracle.attn_bwd_ref(q, k, v, dout, causal, 0.35)
        for b, h in [(0, 0), (1, 3)]:
            Or, Lr = oracle.attn_fwd_rows(q, k, v, causal, 0.35, b, h, rows)
            np.testing.assert_allclose(Or, O[b, h, rows], atol=1e-14)
            np.testing.assert_allclose(Lr, L[b, h, rows], atol=1e-14)
            dqr = oracle.attn_bwd_rows(q, k, v, dout, causal, 0.35, b, h, rows)
            np.testing.assert_allclose(dqr, dq[b, h, rows], atol=1e-13)
        for b, g in [(0, 1), (1, 0)]:
            dkr, dvr = oracle.attn_bwd_kv_rows(q, k, v, dout, causal, 0.35, b, g, rows)
            np.testing.assert_allclose(dkr, dk[b, g, rows], atol=1e-13)
            np.testing.assert_allclose(dvr, dv[b, g, rows], atol=1e-13)


def test_row_chunking_does_not_change_results(monkeypatch):
    q = rnd((1, 2, 50, 4), 131)
    k = rnd((1, 2, 50, 4), 132)
    v = rnd((1, 2, 50, 4), 133)
    dout = rnd((1, 2, 50, 4), 134)
    ref = oracle.attn_fwd_ref(q, k, v, True, 0.5) + oracle.attn_bwd_ref(q, k, v, dout, True, 0.5)
    monkeypatch.setattr(A, "_ROW_CHUNK", 7)
    got = oracle.attn_fwd_ref(q, k, v, True, 0.5) + oracle.attn_bwd_ref(q, k, v, dout, True, 0.5)
    for a, b in zip(ref, got):
        np.testing.assert_allclose(a, b, atol=1e-14)


def test_bad_shapes_raise():
    with pytest.raises(ValueError):
        oracle.attn_fwd_ref(np.zeros((1, 3, 4, 2)), np.zeros((1, 2, 4, 2)), np.zeros((1, 2, 4, 2)), False, 1.0)
    with pytest.raises(ValueError):
        oracle.attn_fwd_ref(np.zeros((1, 2, 4, 2)), np.zeros((1, 2, 5, 2)), np.zeros((1, 2, 5, 2)), False, 1.0)
