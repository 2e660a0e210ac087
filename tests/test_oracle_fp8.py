"""Pins of the FP8 oracle (oracle/fp8.py) against the e4m3 format's
definition, an independent library conversion, quantization invariants, and
the plain attention oracle on exactly representable inputs. Planted mistakes
(on the CPU, in the oracle) must fail at least one pin."""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8 as F


# ----------------------------------------------------------------- format

def test_decode_spot_values_from_the_bit_fields():
    want = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
            0x40: 2.0, 0x7E: 448.0, 0x77: 240.0, 0xB8: -1.0, 0xFE: -448.0}
    got = F.e4m3_decode(np.array(list(want), dtype=np.uint8))
    assert np.array_equal(got, np.array(list(want.values())))
    assert np.isnan(F.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()
    assert F.e4m3_decode(np.array([0x80], dtype=np.uint8))[0] == 0.0


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(F.e4m3_encode(F.e4m3_decode(codes)), codes)
    # The sign of zero is kept: a tiny negative value rounds to 0x80.
    assert np.array_equal(F.e4m3_encode(np.array([-1e-9, 1e-9, -0.0])), np.array([0x80, 0x00, 0x80], np.uint8))


def test_ties_go_to_the_even_code_and_range_saturates():
    x = np.array([1.0625, 1.1875, -1.0625, 2.0 ** -10, 3 * 2.0 ** -10, 500.0, -1e9, 464.0])
    # 1.0625 lies halfway between 1.0 (0x38) and 1.125 (0x39): even code 0x38.
    # 1.1875 between 1.125 (0x39) and 1.25 (0x3A): 0x3A. Half the smallest
    # subnormal ties to 0; 1.5 subnormal steps ties to 2 steps (0x02).
    want = np.array([0x38, 0x3A, 0xB8, 0x00, 0x02, 0x7E, 0xFE, 0x7E], dtype=np.uint8)
    assert np.array_equal(F.e4m3_encode(x), want)


def test_encode_matches_torch_float8_conversion():
    # torch's own e4m3fn cast (round to nearest even) on values inside the
    # finite range, as an independent implementation.
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 200.0)])
    x = np.clip(x, -448.0, 448.0).astype(np.float32).astype(np.float64)
    x = np.concatenate([x, [-1e-7, 1e-7]])  # values that round to -0 and +0
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(x), ref)


# ------------------------------------------------------------- quantization

def _bf16_values(shape, seed, gain=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * gain).to(torch.bfloat16).double().numpy()


def test_block_amax_maps_to_448_and_scale_is_amax_over_448():
    x = _bf16_values((2, 3, 300, 64), 1)
    codes, scales = F.quantize_blocks(x)
    assert scales.shape == (2, 3, 3) and scales.dtype == np.float32
    for idx in np.ndindex(2, 3):
        for b in range(3):
            blk = x[idx][b * 128:(b + 1) * 128]
            amax = np.float32(np.abs(blk).max())
            assert scales[idx + (b,)] == amax / np.float32(448.0)
            i = np.unravel_index(np.abs(blk).argmax(), blk.shape)
            assert F.e4m3_decode(codes[idx][b * 128:(b + 1) * 128][i]) in (448.0, -448.0)


def test_dequantization_error_is_within_half_an_e4m3_step():
    x = _bf16_values((1, 2, 513, 128), 2, gain=3.0)
    codes, scales = F.quantize_blocks(x)
    xh = F.dequantize_blocks(codes, scales)
    s = np.repeat(scales.astype(np.float64), 128, axis=-1)[..., :513, None]
    # Relative 2^-4 for normal codes; absolute 2^-10 * s in the subnormal range,
    # plus the fp32 rounding of the product x * (448 / amax).
    bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * s) * (1 + 2.0 ** -20) + 2.0 ** -22 * s * 448
    assert (np.abs(xh - x) <= bound).all()


def test_per_head_block_and_zero_block():
    x = _bf16_values((1, 2, 200, 64), 3)
    x[0, 1] = 0.0
    codes, scales = F.quantize_blocks(x, None)
    assert scales.shape == (1, 2, 1)
    assert scales[0, 1, 0] == 1.0 and not codes[0, 1].any()
    assert scales[0, 0, 0] == np.float32(np.abs(x[0, 0]).max()) / np.float32(448)


# --------------------------------------------------------------- attention

def _representable(shape, seed, block_rows=128):
    """Codes and scales chosen directly, so the dequantized tensor is known
    exactly (no quantization step involved)."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 0x7F, size=shape).astype(np.uint8)
    codes = np.where(rng.random(shape) < 0.5, codes | 0x80, codes).astype(np.uint8)
    codes = np.where((codes & 0x7F) == 0x7F, 0x7E, codes).astype(np.uint8)
    N = shape[-2]
    nb = 1 if block_rows is None else (N + block_rows - 1) // block_rows
    scales = (2.0 ** rng.integers(-9, -5, size=shape[:-2] + (nb,))).astype(np.float32)
    return codes, scales


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_attention_is_attention_on_the_dequantized_tensors(causal):
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 64
    q8, sq = _representable((B, Hq, N, d), 5)
    k8, sk = _representable((B, Hkv, N, d), 6)
    v8, sv = _representable((B, Hkv, N, d), 7, None)
    O, L = oracle.attn_fwd_fp8_ref(q8, sq, k8, sk, v8, sv, causal, 0.125)
    # The same attention written out from the decoded values and the scales
    # placed by hand: row r of a Q/K head belongs to block r // 128.
    q = F.e4m3_decode(q8) * np.repeat(sq.astype(np.float64), 128, axis=-1)[..., :N, None]
    k = F.e4m3_decode(k8) * np.repeat(sk.astype(np.float64), 128, axis=-1)[..., :N, None]
    v = F.e4m3_decode(v8) * sv.astype(np.float64)[..., None]
    O2, L2 = oracle.attn_fwd_ref(q, k, v, causal, 0.125)
    assert np.abs(O - O2).max() < 1e-12 and np.abs(L - L2).max() < 1e-12


def test_dequantized_attention_tracks_bf16_attention_within_quantization_error():
    B, H, N, d = 1, 2, 256, 64
    q, k, v = (_bf16_values((B, H, N, d), s) for s in (21, 22, 23))
    q8, sq = F.quantize_blocks(q)
    k8, sk = F.quantize_blocks(k)
    v8, sv = F.quantize_blocks(v, None)
    O8, _ = oracle.attn_fwd_fp8_ref(q8, sq, k8, sk, v8, sv, True, d ** -0.5)
    O, _ = oracle.attn_fwd_ref(q, k, v, True, d ** -0.5)
    # FP8 changes rounding (not identical) but stays close: V's own
    # quantization moves O by up to half an e4m3 step, 2^-4 |v| (causal row 0
    # is exactly a dequantized V row), and Q, K's move the scores a little.
    rel = np.abs(O8 - O).max() / np.abs(v).max()
    assert 1e-5 < rel < 2.0 ** -4
    assert np.array_equal(O8[0, :, 0], F.dequantize_blocks(v8, sv, None)[0, :, 0])


# ---------------------------------------------------------- planted mistakes

def _all_pins_pass():
    checks = [test_decode_spot_values_from_the_bit_fields, test_every_finite_code_round_trips,
              test_ties_go_to_the_even_code_and_range_saturates, test_encode_matches_torch_float8_conversion,
              test_block_amax_maps_to_448_and_scale_is_amax_over_448,
              test_dequantization_error_is_within_half_an_e4m3_step,
              lambda: test_fp8_attention_is_attention_on_the_dequantized_tensors(True)]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def test_unmutated_fp8_oracle_passes():
    assert _all_pins_pass()


def test_mutation_wrong_exponent_bias_is_caught(monkeypatch):
    orig = F.e4m3_decode
    monkeypatch.setattr(F, "e4m3_decode", lambda c: orig(c) * 2.0)
    assert not _all_pins_pass()


def test_mutation_ties_away_from_zero_is_caught(monkeypatch):
    def enc(x):
        x = np.asarray(x, dtype=np.float64)
        vals, codes = F._positive_grid()
        a = np.minimum(np.abs(x), 448.0)
        idx = np.abs(vals[None, :] - a.reshape(-1, 1))
        best = np.argmin(idx[:, ::-1], axis=1)  # prefers the larger value on ties
        out = codes[len(vals) - 1 - best].reshape(a.shape).astype(np.uint8)
        return np.where(np.signbit(x), out | 0x80, out).astype(np.uint8)
    monkeypatch.setattr(F, "e4m3_encode", enc)
    assert not _all_pins_pass()


def test_mutation_scale_block_off_by_one_row_is_caught(monkeypatch):
    orig = F.dequantize_blocks

    def deq(codes, scales, block_rows=128):
        if block_rows is None:
            return orig(codes, scales, None)
        v = F.e4m3_decode(codes)
        N = v.shape[-2]
        s = np.repeat(np.asarray(scales, dtype=np.float64), block_rows, axis=-1)
        s = np.concatenate([s[..., :1], s], axis=-1)[..., :N]  # rows shifted by one
        return v * s[..., None]
    monkeypatch.setattr(F, "dequantize_blocks", deq)
    assert not _all_pins_pass()
