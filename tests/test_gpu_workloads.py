"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (forward with the O residual, then the backward that uses
it), and for the plain pair fa_fwd / fa_bwd (no residual: the backward forms
D from the bf16 o). Outputs the oracle can afford are compared element by
element: every row for the 2048-token workload, seeded samples of rows for
the longer ones.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_56_b200 import WORKLOADS, fa, sample_rows, to_f64, workload_inputs

from .parity import assert_close_abs, assert_close_lse

pytestmark = pytest.mark.gpu


def _run(w, residual=True):
    host = workload_inputs(w)
    dev = {k: v.cuda() for k, v in host.items()}
    out = {}
    if w.backward:
        if residual:
            o, lse, r = fa.attention_forward(dev["q"], dev["k"], dev["v"], w.causal, w.scale, residual=True)
        else:
            (o, lse), r = fa.attention_forward(dev["q"], dev["k"], dev["v"], w.causal, w.scale), None
        dq, dk, dv = fa.attention_backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, w.causal, w.scale,
                                           o_resid=r)
        out.update(dq=dq.cpu(), dk=dk.cpu(), dv=dv.cpu())
    else:
        o, lse = fa.attention_forward(dev["q"], dev["k"], dev["v"], w.causal, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == fa.FA_OK
    out.update(o=o.cpu(), lse=lse.cpu())
    del dev
    torch.cuda.empty_cache()
    return host, out


def _head(host, name, b, h):
    return to_f64(host[name][b:b + 1, h:h + 1])


@pytest.mark.parametrize("residual", [True, False], ids=["with_residual", "plain_pair"])
@pytest.mark.parametrize("name", ["fwdbwd_b4_h16_n2048_d64_causal", "fwdbwd_b4_h16_n2048_d64"])
def test_b4_h16_n2048_d64_all_rows(name, residual):
    # plain_pair: fa_fwd then fa_bwd, the boundary's own signatures.
    w = WORKLOADS[name]
    host, out = _run(w, residual)
    ref = {k: to_f64(v) for k, v in host.items()}
    O, L = oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], w.causal, w.scale)
    assert_close_abs("O", to_f64(out["o"]), O)
    assert_close_lse(to_f64(out["lse"]), L)
    gq, gk, gv = oracle.attn_bwd_ref(ref["q"], ref["k"], ref["v"], ref["dout"], w.causal, w.scale)
    assert_close_abs("dQ", to_f64(out["dq"]), gq)
    assert_close_abs("dK", to_f64(out["dk"]), gk)
    assert_close_abs("dV", to_f64(out["dv"]), gv)


def _probs(q, k, causal, scale, rows):
    """Softmax rows P [len(rows), N] of one head (plain numpy, fp64)."""
    S = scale * (q[rows] @ k.T)
    if causal:
        S[np.arange(k.shape[0])[None, :] > np.asarray(rows)[:, None]] = -np.inf
    P = np.exp(S - S.max(axis=1, keepdims=True))
    return P / P.sum(axis=1, keepdims=True)


def _d_error_bound(P, v, do, O):
    """Bound on |D_i(o) - D_i(O)| when D is formed from the bf16 o instead of
    the exact O. The kernel's O before rounding differs from the exact one by
    the bf16 rounding of the weights P (at most 2^-8 P_k |V_k| summed), and
    rounding it to the bf16 o adds at most 2^-8 |O|; D_i = sum_c dO_ic o_ic
    sums those errors times |dO|."""
    return 2.0 ** -8 * (np.abs(do) * (P @ np.abs(v) + np.abs(O))).sum(axis=1)


def _check_sampled(w, rows_per_head, kv_rows=None, kv_groups=(), residual=True):
    """Sampled rows of O, L, dQ for every (batch, head), and dK, dV rows of
    the listed (batch, KV head) groups. Without the residual (the plain
    fa_fwd / fa_bwd pair) the gradients may also carry the error of D formed
    from the bf16 o; that error is bounded from the oracle's own P and O
    (``_d_error_bound``) and added to the tolerance of dQ and dK (dV does
    not depend on D)."""
    host, out = _run(w, residual)
    r = w.Hq // w.Hkv
    for b in range(w.B):
        for h in range(w.Hq):
            rows = sample_rows(w.N, rows_per_head, w.seed * 131 + b * 977 + h)
            g = h // r
            q, k, v = _head(host, "q", b, h), _head(host, "k", b, g), _head(host, "v", b, g)
            O, L = oracle.attn_fwd_rows(q, k, v, w.causal, w.scale, 0, 0, rows)
            assert_close_abs(f"O[{b},{h}]", to_f64(out["o"][b, h, rows]), O)
            assert_close_lse(to_f64(out["lse"][b, h, rows]), L)
            if w.backward:
                do = _head(host, "dout", b, h)
                dq = oracle.attn_bwd_rows(q, k, v, do, w.causal, w.scale, 0, 0, rows)
                extra = 0.0
                if not residual:
                    P = _probs(q[0, 0], k[0, 0], w.causal, w.scale, rows)
                    dD = _d_error_bound(P, v[0, 0], do[0, 0, rows], O)
                    extra = w.scale * dD[:, None] * (P @ np.abs(k[0, 0]))
                assert_close_abs(f"dQ[{b},{h}]", to_f64(out["dq"][b, h, rows]), dq, extra=extra)
    if not w.backward:
        return
    for (b, g) in kv_groups:
        heads = slice(g * r, (g + 1) * r)
        q = to_f64(host["q"][b:b + 1, heads])
        do = to_f64(host["dout"][b:b + 1, heads])
        k, v = _head(host, "k", b, g), _head(host, "v", b, g)
        keys = np.arange(w.N) if kv_rows is None else sample_rows(w.N, kv_rows, w.seed * 7 + b * 31 + g)
        dk, dv = oracle.attn_bwd_kv_rows(q, k, v, do, w.causal, w.scale, 0, 0, keys)
        extra = 0.0
        if not residual:
            extra = np.zeros((len(keys), w.d))
            for hh in range(r):
                qh = q[0, hh]
                O, _ = oracle.attn_fwd_rows(q[:, hh:hh + 1], k, v, w.causal, w.scale, 0, 0, np.arange(w.N))
                for r0 in range(0, w.N, 512):
                    rr = np.arange(r0, min(w.N, r0 + 512))
                    P = _probs(qh, k[0, 0], w.causal, w.scale, rr)
                    dD = _d_error_bound(P, v[0, 0], do[0, hh, rr], O[rr])
                    extra += w.scale * (P[:, keys] * dD[:, None]).T @ np.abs(qh[rr])
        assert_close_abs(f"dK[{b},{g}]", to_f64(out["dk"][b, g, keys]), dk, extra=extra)
        assert_close_abs(f"dV[{b},{g}]", to_f64(out["dv"][b, g, keys]), dv)


def test_b2_h16_n8192_d128_causal_peaky_sampled():
    # 256 seeded query rows per head for O, L, dQ; every key row of dK, dV
    # for two (batch, head) slices.
    w = WORKLOADS["fwdbwd_b2_h16_n8192_d128_causal_peaky"]
    _check_sampled(w, 256, kv_groups=[(0, 3), (1, 12)])


def test_b2_h16_n8192_d128_causal_peaky_plain_pair_sampled():
    # The boundary's own pair (fa_fwd, then fa_bwd with D from the bf16 o) on
    # the same rows: O and L within the plain tolerance, dQ and dK within it
    # plus the derived bound on the error D carries in from the bf16 o.
    w = WORKLOADS["fwdbwd_b2_h16_n8192_d128_causal_peaky"]
    _check_sampled(w, 256, kv_groups=[(0, 3), (1, 12)], residual=False)


def test_gqa_b1_hq32_hkv8_n16384_d128_causal_sampled():
    # 128 seeded query rows per query head for O, L, dQ; 128 seeded key rows
    # of dK, dV for one KV group (its four query heads rebuilt in full).
    w = WORKLOADS["fwdbwd_gqa_b1_hq32_hkv8_n16384_d128_causal"]
    _check_sampled(w, 128, kv_rows=128, kv_groups=[(0, 5)])


def test_b1_h8_n131072_d128_causal_fwd_sampled_and_no_nxn_buffer():
    w = WORKLOADS["fwd_b1_h8_n131072_d128_causal"]
    host = workload_inputs(w)
    dev = {k: v.cuda() for k, v in host.items()}
    o = torch.empty_like(dev["q"])
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    fa.fa_fwd(dev["q"], dev["k"], dev["v"], o, lse, w.causal, w.scale)  # loads the module
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base_alloc = torch.cuda.memory_allocated()
    free_before, _ = torch.cuda.mem_get_info()
    fa.fa_fwd(dev["q"], dev["k"], dev["v"], o, lse, w.causal, w.scale)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert fa.fa_check_device_error() == fa.FA_OK
    # Nothing is allocated by the call: a naive fp32 score matrix here would
    # be 8 * 131072^2 * 4 B = 512 GiB; the bound is 64 MiB.
    assert torch.cuda.max_memory_allocated() - base_alloc <= 64 << 20
    assert free_before - free_after <= 64 << 20
    out_o, out_l = o.cpu(), lse.cpu()
    del dev, o, lse
    torch.cuda.empty_cache()
    for h in range(w.Hq):
        rows = sample_rows(w.N, 64, w.seed * 131 + h)
        q, k, v = _head(host, "q", 0, h), _head(host, "k", 0, h), _head(host, "v", 0, h)
        O, L = oracle.attn_fwd_rows(q, k, v, w.causal, w.scale, 0, 0, rows)
        assert_close_abs(f"O[{h}]", to_f64(out_o[0, h, rows]), O)
        assert_close_lse(to_f64(out_l[0, h, rows]), L)
