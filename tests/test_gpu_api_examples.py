"""The convenience calls of the Python binding (attention_forward,
attention_backward, attention_decode, attention_forward_fp8) used the way a
caller would, at a smaller N, checked against the oracle."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_56_b200 import fa, to_f64

from .parity import assert_close_abs, assert_close_lse

pytestmark = pytest.mark.gpu


def test_convenience_calls_against_the_oracle():
    g = torch.Generator().manual_seed(12)
    q = torch.randn(2, 16, 384, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(2, 4, 384, 128, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(2, 4, 384, 128, generator=g).to(torch.bfloat16).cuda()
    dout = torch.randn(2, 16, 384, 128, generator=g).to(torch.bfloat16).cuda()
    ref = {n: to_f64(t) for n, t in (("q", q), ("k", k), ("v", v), ("dout", dout))}
    scale = 128 ** -0.5

    o, lse, o_resid = fa.attention_forward(q, k, v, causal=True, residual=True)
    dq, dk, dv = fa.attention_backward(q, k, v, o, dout, lse, causal=True, o_resid=o_resid)
    torch.cuda.synchronize()
    O, L = oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], True, scale)
    assert_close_abs("O", to_f64(o), O)
    assert_close_lse(to_f64(lse), L)
    gq, gk, gv = oracle.attn_bwd_ref(ref["q"], ref["k"], ref["v"], ref["dout"], True, scale)
    for name, got, want in (("dQ", dq, gq), ("dK", dk, gk), ("dV", dv, gv)):
        assert_close_abs(name, to_f64(got), want)

    o, lse = fa.attention_forward(q, k, v, causal=True, window=100, prefix=16)
    O, L = oracle.attn_fwd_ref(ref["q"], ref["k"], ref["v"], True, scale, 100, 16)
    assert_close_abs("O masked", to_f64(o), O)

    od, ld = fa.attention_decode(q[:, :, -1:].contiguous(), k, v)
    Od, Ld = oracle.attn_decode_ref(ref["q"][:, :, -1:], ref["k"], ref["v"], scale, True)
    assert_close_abs("O decode", to_f64(od), Od)
    assert_close_lse(to_f64(ld), Ld)

    o8, l8, (q8, sq, k8, sk, v8, sv) = fa.attention_forward_fp8(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == fa.FA_OK
    # The codes the call produced are the quantizer's; the forward is checked
    # against the oracle's quantization of the same inputs (bit-identical).
    wq8, wsq = oracle.quantize_blocks(ref["q"])
    assert np.array_equal(q8.cpu().numpy(), wq8) and np.array_equal(sq.cpu().numpy().reshape(wsq.shape), wsq)
    wk8, wsk = oracle.quantize_blocks(ref["k"])
    wv8, wsv = oracle.quantize_blocks(ref["v"], None)
    O8, L8 = oracle.attn_fwd_fp8_ref(wq8, wsq, wk8, wsk, wv8, wsv, True, scale)
    vh = oracle.dequantize_blocks(wv8, wsv, None)
    assert (np.abs(to_f64(o8) - O8) <= 2.0 ** -4 * np.abs(vh).max() + 2.0 ** -8 * np.abs(O8)).all()
    assert_close_lse(to_f64(l8), L8)
