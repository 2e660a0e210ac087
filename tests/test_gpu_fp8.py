"""GPU checks of the FP8 mode: the e4m3 block quantizer against the oracle's
(bit for bit: codes and scales), and the FP8 forward against exact attention
on the dequantized tensors, within a bound derived from its arithmetic.

Tolerance of the forward. Both products take e4m3 operands; Q, K, V enter
as given (the oracle dequantizes the same codes), so the kernel's own
rounding is: the softmax weights enter the second product as e4m3 of
w = 2^(x + 4), x the exponent against a running max that may lag the true
one by up to 4 (so w <= 2^8 and the row's largest w >= 2^4, hence the sum
of w >= 2^4). e4m3 moves w by at most 2^-4 w (half a step of a 3-bit
mantissa) or, in its subnormal range, 2^-10; in units of the normalised
weight P = w / sum(w) that is 2^-4 P or 2^-10 / 2^4 = 2^-14. Hence, element
by element,
    |O - O_ref| <= 2^-4 (P |V|) + 2^-14 sum_k |V_k| + 2^-8 |O_ref| + 1e-5 max|V|
(last two: the bf16 output's rounding and fp32 accumulation). The mean error
must also stay well below the mean bound (rounding errors of random sign
average out). L: |dL| <= 1e-3 max(1, |L|) as for bf16 (l sums unrounded
weights)."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_56_b200 import fa, make_inputs, sample_rows, to_f64

from .parity import assert_close_lse

pytestmark = pytest.mark.gpu


def quantized_inputs(B, Hq, Hkv, N, d, seed, qk_gain=1.0):
    """bf16 inputs quantized by the oracle (CPU): codes and scales for both
    the GPU call and the oracle."""
    host = make_inputs(B, Hq, Hkv, N, d, seed, qk_gain, with_dout=False)
    q8, sq = oracle.quantize_blocks(to_f64(host["q"]))
    k8, sk = oracle.quantize_blocks(to_f64(host["k"]))
    v8, sv = oracle.quantize_blocks(to_f64(host["v"]), None)
    return {"q8": q8, "sq": sq, "k8": k8, "sk": sk, "v8": v8, "sv": sv}


def run_fp8(qi, causal, scale):
    B, Hq, N, d = qi["q8"].shape
    Hkv = qi["k8"].shape[1]
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in qi.items()}
    o = torch.empty(B, Hq, N, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device="cuda")
    fa.fa_fwd_fp8(t["q8"], t["sq"].reshape(B * Hq, -1), t["k8"], t["sk"].reshape(B * Hkv, -1), t["v8"],
                  t["sv"].reshape(B * Hkv), o, lse, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == fa.FA_OK
    return to_f64(o), to_f64(lse)


def fp8_bound(qh, kh, vh, causal, scale, O_ref, rows=None):
    """Elementwise error bound of the module docstring, per (b, h, row, col)."""
    B, Hq, N, d = qh.shape
    r = Hq // kh.shape[1]
    rows = np.arange(N) if rows is None else rows
    out = np.empty((B, Hq, len(rows), d))
    for b in range(B):
        for h in range(Hq):
            k, v = kh[b, h // r], vh[b, h // r]
            S = scale * qh[b, h, rows] @ k.T
            if causal:
                S[np.arange(N)[None, :] > rows[:, None]] = -np.inf
            P = np.exp(S - S.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            out[b, h] = 2.0 ** -4 * (P @ np.abs(v)) + 2.0 ** -14 * np.abs(v).sum(axis=0)
    return out + 2.0 ** -8 * np.abs(O_ref) + 1e-5 * np.abs(vh).max()


def check_fp8(B, Hq, Hkv, N, d, causal, seed, qk_gain=1.0):
    qi = quantized_inputs(B, Hq, Hkv, N, d, seed, qk_gain)
    scale = d ** -0.5
    o, lse = run_fp8(qi, causal, scale)
    O, L = oracle.attn_fwd_fp8_ref(qi["q8"], qi["sq"], qi["k8"], qi["sk"], qi["v8"], qi["sv"], causal, scale)
    qh = oracle.dequantize_blocks(qi["q8"], qi["sq"])
    kh = oracle.dequantize_blocks(qi["k8"], qi["sk"])
    vh = oracle.dequantize_blocks(qi["v8"], qi["sv"], None)
    bound = fp8_bound(qh, kh, vh, causal, scale, O)
    err = np.abs(o - O)
    assert np.isfinite(o).all()
    assert (err <= bound).all(), f"max excess {(err - bound).max():.3e}, max err {err.max():.3e}"
    assert err.mean() <= 0.25 * bound.mean(), (err.mean(), bound.mean())
    assert_close_lse(lse, L)


# ------------------------------------------------------------- quantizer

@pytest.mark.parametrize("N", [1, 127, 129, 300])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("per_head", [False, True])
def test_quantizer_matches_oracle_bit_for_bit(N, d, per_head):
    host = make_inputs(2, 3, 3, N, d, 40 + N + d, 3.0, with_dout=False)
    x = host["q"].clone()
    x[1, 2] = 0.0                # an all-zero head (and, per block, all-zero blocks)
    x[0, 0, 0, :4] = -0.0        # negative zeros inside a nonzero block
    codes, scales = fa.quantize_fp8(x.cuda(), per_head)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == fa.FA_OK
    want_c, want_s = oracle.quantize_blocks(to_f64(x), None if per_head else 128)
    assert np.array_equal(codes.cpu().numpy(), want_c)
    assert np.array_equal(scales.cpu().numpy().reshape(want_s.shape), want_s)


# ------------------------------------------------------------------ forward

@pytest.mark.parametrize("N,causal", [(1, True), (129, False), (300, True), (300, False), (1024, True)])
def test_fp8_forward_shapes(N, causal):
    check_fp8(1, 2, 2, N, 128, causal, seed=700 + N)


@pytest.mark.parametrize("ratio", [2, 4])
def test_fp8_forward_gqa(ratio):
    check_fp8(2, 2 * ratio, 2, 640, 128, True, seed=720 + ratio)


def test_fp8_forward_peaky():
    check_fp8(1, 2, 1, 768, 128, True, seed=731, qk_gain=2.0)


def test_fp8_forward_saturated_rows():
    # One key per row dominates by far more than the fp32 underflow gap: its
    # weight (a power of two) is exact in e4m3, so O is that key's
    # dequantized V row up to the bf16 output rounding and the last-bit error
    # of l.
    B, H, N, d = 1, 2, 400, 128
    g = torch.Generator().manual_seed(77)
    kc = torch.randint(0, 2, (B, H, N, d), generator=g) * 2 - 1
    k8 = np.where(kc.numpy() > 0, 0x38, 0xB8).astype(np.uint8)          # +-1.0
    rng = np.random.default_rng(77)
    pick = np.array([[rng.integers(0, i + 1) for i in range(N)] for _ in range(H)])
    q8 = np.stack([k8[0, h][pick[h]] for h in range(H)])[None].copy()
    q8 = np.where(q8 == 0x38, 0x70, 0xF0).astype(np.uint8)               # +-128 (exponent field 14)
    nb = (N + 127) // 128
    sq = np.full((B, H, nb), 0.5, np.float32)                            # so q = 64 * k
    sk = np.ones((B, H, nb), np.float32)
    v = make_inputs(B, H, H, N, d, 78, with_dout=False)["v"]
    v8, sv = oracle.quantize_blocks(to_f64(v), None)
    kh = oracle.dequantize_blocks(k8, sk)
    gap = d - max(np.max(np.where(np.eye(N, dtype=bool), -np.inf, kh[0, h] @ kh[0, h].T)) for h in range(H))
    assert 64 * d ** -0.5 * np.log2(np.e) * gap > 160
    o, _ = run_fp8({"q8": q8, "sq": sq, "k8": k8, "sk": sk, "v8": v8, "sv": sv}, True, d ** -0.5)
    vh = oracle.dequantize_blocks(v8, sv, None)
    for h in range(H):
        want = vh[0, h][pick[h]]
        assert (np.abs(o[0, h] - want) <= 2.0 ** -8 * np.abs(want) + 1e-6).all(), h


def test_fp8_forward_full_workload_sampled_rows():
    # The headline shape in FP8 mode: B=2, H=16, N=8192, d=128, causal, Q/K gain 2.
    B, H, N, d = 2, 16, 8192, 128
    qi = quantized_inputs(B, H, H, N, d, 1002, 2.0)
    scale = d ** -0.5
    o, lse = run_fp8(qi, True, scale)
    qh = oracle.dequantize_blocks(qi["q8"], qi["sq"])
    kh = oracle.dequantize_blocks(qi["k8"], qi["sk"])
    vh = oracle.dequantize_blocks(qi["v8"], qi["sv"], None)
    for b, h in ((0, 0), (1, 15)):
        rows = sample_rows(N, 64, 1002 + 17 * b + h)
        O, L = oracle.attn_fwd_rows(qh, kh, vh, True, scale, b, h, rows)
        bound = fp8_bound(qh[b:b + 1, h:h + 1], kh[b:b + 1, h:h + 1], vh[b:b + 1, h:h + 1], True, scale,
                          O[None, None], rows)[0, 0]
        err = np.abs(o[b, h, rows] - O)
        assert (err <= bound).all(), (b, h, (err - bound).max())
        assert_close_lse(lse[b, h, rows], L)


def test_fp8_argument_errors():
    qi = quantized_inputs(1, 1, 1, 64, 128, 1)
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in qi.items()}
    o = torch.empty(1, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, 1, 64, device="cuda")
    with pytest.raises(fa.FaError):
        fa.fa_fwd_fp8(t["q8"], t["sq"].reshape(1, -1), t["k8"], t["sk"].reshape(1, -1), t["v8"],
                      t["sv"].reshape(1), o, lse, True, float("inf"))
    x64 = torch.zeros(1, 1, 64, 64, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FaError):  # d = 64 is not an FP8 forward shape
        fa.fa_fwd_fp8(x64, t["sq"].reshape(1, -1), x64, t["sk"].reshape(1, -1), x64, t["sv"].reshape(1),
                      torch.empty(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda"), lse, True, 0.1)
