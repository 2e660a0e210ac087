"""Planted mistakes in the oracle must be caught by its pins.

Each mutation patches the oracle on the CPU (never the CUDA path) with a
plausible error: an off-by-one causal mask, a dropped scale, a missing
normalisation, the wrong logarithm base, a flipped sign, swapped or
mis-summed gradients. The test passes only if at least one pin in
``test_oracle_pins`` fails under the mutation.
"""

import numpy as np
import pytest

import oracle
from oracle import attention as A

from . import test_oracle_pins as pins

FWD_CHECKS = [pins.check_brute_force, pins.check_online_equals_two_pass, pins.check_rows_sum_to_one,
              pins.check_constant_v, pins.check_zero_q, pins.check_causal_row0,
              pins.check_permutation_invariance]


def _fails(checks, **kw):
    for c in checks:
        try:
            c(**kw)
        except AssertionError:
            return True
    return False


_orig_scores = A._scores
_orig_softmax = A._softmax_rows


def scores_mask_off_by_one(qrows, kmat, scale, causal, row_ids, window=None, prefix=0):
    S = scale * (qrows @ kmat.T)
    if causal:
        cols = np.arange(kmat.shape[0])
        S[cols[None, :] >= np.asarray(row_ids)[:, None] + 2] = -np.inf
    return S


def scores_no_scale(qrows, kmat, scale, causal, row_ids, window=None, prefix=0):
    return _orig_scores(qrows, kmat, 1.0, causal, row_ids, window, prefix)


def scores_transposed(qrows, kmat, scale, causal, row_ids, window=None, prefix=0):
    # Uses K's rows in reverse order (a wrong index into K).
    return _orig_scores(qrows, kmat[::-1], scale, causal, row_ids, window, prefix)


def softmax_unnormalised(S):
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    return E, (m + np.log(E.sum(axis=1, keepdims=True)))[:, 0]


def softmax_log2(S):
    P, L = _orig_softmax(S)
    return P, L / np.log(2.0)


@pytest.mark.parametrize("name,target,repl", [
    ("causal mask off by one", "_scores", scores_mask_off_by_one),
    ("scale dropped", "_scores", scores_no_scale),
    ("key rows misindexed", "_scores", scores_transposed),
    ("softmax not normalised", "_softmax_rows", softmax_unnormalised),
    ("logsumexp in base 2", "_softmax_rows", softmax_log2),
])
def test_forward_mutation_is_caught(monkeypatch, name, target, repl):
    monkeypatch.setattr(A, target, repl)
    assert _fails(FWD_CHECKS), name


_orig_merge = A.merge_softmax_states


def merge_second_not_rescaled(a, b):
    # Forgets to bring the second state to the common maximum.
    ma, la, Ua = a
    mb, lb, Ub = b
    M = np.maximum(ma, mb)
    ref = np.where(np.isneginf(M), 0.0, M)
    fa = np.where(np.isneginf(ma), 0.0, np.exp(ma - ref))
    fb = np.where(np.isneginf(mb), 0.0, 1.0)
    return M, fa * la + fb * lb, fa[:, None] * Ua + fb[:, None] * Ub


def merge_output_not_rescaled(a, b):
    # Rescales the sums but not the partial outputs.
    M, l, _ = _orig_merge(a, b)
    return M, l, a[2] + b[2]


def merge_sign_flipped(a, b):
    # e^(M - m) instead of e^(m - M).
    ma, la, Ua = a
    mb, lb, Ub = b
    M = np.maximum(ma, mb)
    ref = np.where(np.isneginf(M), 0.0, M)
    fa = np.where(np.isneginf(ma), 0.0, np.exp(ref - ma))
    fb = np.where(np.isneginf(mb), 0.0, np.exp(ref - mb))
    return M, fa * la + fb * lb, fa[:, None] * Ua + fb[:, None] * Ub


@pytest.mark.parametrize("name,repl", [
    ("second state not rescaled", merge_second_not_rescaled),
    ("partial outputs not rescaled", merge_output_not_rescaled),
    ("rescale exponent sign flipped", merge_sign_flipped),
])
def test_merge_mutation_is_caught(monkeypatch, name, repl):
    monkeypatch.setattr(A, "merge_softmax_states", repl)
    monkeypatch.setattr(oracle, "merge_softmax_states", repl)
    assert _fails([pins.check_online_equals_two_pass, pins.check_online_any_merge_order,
                   pins.check_merge_closed_form]), name


def _wrap_bwd(kind):
    ref = oracle.attn_bwd_ref

    def bwd(q, k, v, dout, causal, scale):
        dq, dk, dv = ref(q, k, v, dout, causal, scale)
        if kind == "dq sign":
            return -dq, dk, dv
        if kind == "dk no scale":
            return dq, dk / scale, dv
        if kind == "dk dv swapped":
            return dq, dv, dk
        if kind == "gqa not summed":
            # Keeps only the first query head's share of each KV head.
            r = q.shape[1] // k.shape[1]
            if r == 1:
                return dq, dk, dv
            q1 = q.copy(); dout1 = dout.copy()
            for h in range(q.shape[1]):
                if h % r:
                    dout1[:, h] = 0.0
            _, dk1, dv1 = ref(q1, k, v, dout1, causal, scale)
            return dq, dk1, dv1
        raise KeyError(kind)
    return bwd


@pytest.mark.parametrize("kind", ["dq sign", "dk no scale", "dk dv swapped", "gqa not summed"])
def test_backward_mutation_is_caught(kind):
    assert _fails([pins.check_backward_fd], bwd=_wrap_bwd(kind)), kind


def test_unmutated_oracle_passes_all_checks():
    assert not _fails(FWD_CHECKS + [pins.check_backward_fd])
