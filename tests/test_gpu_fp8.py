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
weight P = w / sum(w) that is 2^-4 P or min(P, 2^-10 / 2^4 = 2^-14); only keys
whose exact relative weight e^(S_k - max S) is below 2^-10 can be subnormal.
Hence, element by element,
    |O - O_ref| <= E + 2^-8 (|O_ref| + E) + 1e-5 max|V|,  E = sum_k e_k |V_k|,
    e_k = 2^-4 P_k, or max(2^-4 P_k, min(P_k, 2^-14)) for those keys
(last two: the bf16 rounding of the kernel's value, which lies within E of
O_ref, and fp32 accumulation). The mean error
must also stay well below the mean bound (rounding errors of random sign
average out). L: |dL| <= 1e-3 max(1, |L|) as for bf16 (l sums unrounded
weights)."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_56_b200 import FP8_WORKLOADS, fa, make_inputs, sample_rows, to_f64

from .parity import assert_close_lse, record_bound

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
    """Elementwise error bound of the module docstring, per (b, h, row, col).

    Per key k with exact weight P_k and u_k = e^(S_k - max S): a key with
    u_k >= 2^-10 always has w >= 2^4 u_k >= 2^-6, a normal e4m3 value, so
    its normalised weight moves by at most 2^-4 P_k; only a key with
    u_k < 2^-10 can fall into the subnormal range, where the move is at most
    min(w, 2^-10) in tile units, i.e. min(P_k, 2^-14) normalised (so at most
    max(2^-4 P_k, min(P_k, 2^-14)))."""
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
            U = np.exp(S - S.max(axis=1, keepdims=True))
            P = U / U.sum(axis=1, keepdims=True)
            E = np.where(U >= 2.0 ** -10, 2.0 ** -4 * P, np.maximum(2.0 ** -4 * P, np.minimum(P, 2.0 ** -14)))
            out[b, h] = E @ np.abs(v)
    # The bf16 output rounds the kernel's value, which may already sit `out`
    # away from O_ref: half an ulp of |O_ref| + out.
    return out + 2.0 ** -8 * (np.abs(O_ref) + out) + 1e-5 * np.abs(vh).max()


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


def _check_fp8_workload(name, rows_per_head):
    """The FP8 bench workload at full size, every (batch, head): seeded
    sampled query rows against exact attention on the dequantized tensors,
    within the elementwise bound of the module docstring (mean error too)."""
    w = FP8_WORKLOADS[name]
    qi = quantized_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, w.qk_gain)
    o, lse = run_fp8(qi, w.causal, w.scale)
    qh = oracle.dequantize_blocks(qi["q8"], qi["sq"])
    kh = oracle.dequantize_blocks(qi["k8"], qi["sk"])
    vh = oracle.dequantize_blocks(qi["v8"], qi["sv"], None)
    del qi
    r = w.Hq // w.Hkv
    errs, bounds = [], []
    for b in range(w.B):
        for h in range(w.Hq):
            rows = sample_rows(w.N, rows_per_head, w.seed * 131 + b * 977 + h)
            g = h // r
            O, L = oracle.attn_fwd_rows(qh, kh, vh, w.causal, w.scale, b, h, rows)
            bound = fp8_bound(qh[b:b + 1, h:h + 1], kh[b:b + 1, g:g + 1], vh[b:b + 1, g:g + 1], w.causal, w.scale,
                              O[None, None], rows)[0, 0]
            err = np.abs(o[b, h, rows] - O)
            record_bound(f"O[{b},{h}]", err, O, bound)
            assert np.isfinite(o[b, h, rows]).all(), (b, h)
            assert (err <= bound).all(), (b, h, float((err - bound).max()), float(err.max()))
            assert_close_lse(lse[b, h, rows], L)
            errs.append(err)
            bounds.append(bound)
    err, bound = np.concatenate(errs), np.concatenate(bounds)
    assert err.mean() <= 0.25 * bound.mean(), (err.mean(), bound.mean())


def test_fp8_workload_b2_h16_n8192_causal_peaky_all_heads():
    # The FP8 bench shape: B=2, H=16, N=8192, d=128, causal, Q/K gain 2 (the
    # lazy rescale acts over up to 64 key tiles per row here).
    _check_fp8_workload("fwd_fp8_b2_h16_n8192_d128_causal_peaky", 64)


def test_fp8_workload_gqa_b1_hq32_hkv8_n16384_causal_all_heads():
    # The FP8 GQA bench shape: B=1, Hq=32, Hkv=8, N=16384, d=128, causal.
    _check_fp8_workload("fwd_fp8_gqa_b1_hq32_hkv8_n16384_d128_causal", 32)


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
