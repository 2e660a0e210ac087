"""Pins of the oracle's decode (short-query) attention."""

import math

import numpy as np
import pytest

import oracle
from oracle import attention as A

from .test_oracle_pins import rnd


def test_decode_equals_last_rows_of_full_causal():
    # The last Nq rows of causal attention over N keys are decode with Nq queries.
    q, k, v = rnd((2, 4, 30, 5), 301, 2.0), rnd((2, 2, 30, 5), 302, 2.0), rnd((2, 2, 30, 5), 303)
    O, L = oracle.attn_fwd_ref(q, k, v, True, 0.6)
    for nq in (1, 3, 30):
        Od, Ld = oracle.attn_decode_ref(q[:, :, -nq:], k, v, 0.6)
        np.testing.assert_allclose(Od, O[:, :, -nq:], atol=1e-14)
        np.testing.assert_allclose(Ld, L[:, :, -nq:], atol=1e-14)


def test_single_query_sees_every_key_brute_force():
    q, k, v = rnd((1, 2, 1, 3), 311), rnd((1, 1, 9, 3), 312), rnd((1, 1, 9, 3), 313)
    O, L = oracle.attn_decode_ref(q, k, v, 0.9)
    for h in range(2):
        s = [0.9 * math.fsum(q[0, h, 0, c] * k[0, 0, j, c] for c in range(3)) for j in range(9)]
        e = [math.exp(x) for x in s]
        assert abs(L[0, h, 0] - math.log(math.fsum(e))) < 1e-14
        for c in range(3):
            assert abs(O[0, h, 0, c] - math.fsum(e[j] * v[0, 0, j, c] for j in range(9)) / math.fsum(e)) < 1e-14


def test_decode_zero_query_is_mean_of_cache():
    v = rnd((1, 1, 17, 4), 321)
    O, L = oracle.attn_decode_ref(np.zeros((1, 1, 1, 4)), rnd((1, 1, 17, 4), 322), v, 1.0)
    np.testing.assert_allclose(O[0, 0, 0], v[0, 0].mean(0), atol=1e-15)
    assert abs(L[0, 0, 0] - math.log(17)) < 1e-15


# --------------------------------------------------------------- mutations
# Planted mistakes in the decode oracle (CPU only): each must make at least
# one of the pins above fail.

PINS = [test_decode_equals_last_rows_of_full_causal, test_single_query_sees_every_key_brute_force,
        test_decode_zero_query_is_mean_of_cache]


def _mutated_decode(kind):
    def decode(q, k, v, scale, causal=True):
        B, Hq, Nq, d = q.shape
        Hkv, Nk = k.shape[1], k.shape[2]
        pos = np.arange(Nk - Nq, Nk)
        if kind == "top-left alignment":
            pos = np.arange(Nq)
        elif kind == "alignment off by one":
            pos = pos - 1
        O = np.empty((B, Hq, Nq, d))
        L = np.empty((B, Hq, Nq))
        for b in range(B):
            for h in range(Hq):
                g = h % Hkv if kind == "kv head by modulo" else A.kv_head_of(h, Hq, Hkv)
                S = A._scores(q[b, h], k[b, g], 1.0 if kind == "scale dropped" else scale, causal, pos)
                P, Lr = A._softmax_rows(S)
                if kind == "not normalised":
                    P = np.exp(S - S.max(axis=1, keepdims=True))
                O[b, h] = P @ v[b, g]
                L[b, h] = Lr
        return O, L
    return decode


def _some_pin_fails():
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("kind", ["top-left alignment", "alignment off by one", "kv head by modulo",
                                  "scale dropped", "not normalised"])
def test_decode_mutation_is_caught(monkeypatch, kind):
    monkeypatch.setattr(oracle, "attn_decode_ref", _mutated_decode(kind))
    assert _some_pin_fails(), kind


def test_unmutated_decode_reimplementation_passes(monkeypatch):
    # The mutation harness itself, with no mutation, passes every pin.
    monkeypatch.setattr(oracle, "attn_decode_ref", _mutated_decode("none"))
    assert not _some_pin_fails()
