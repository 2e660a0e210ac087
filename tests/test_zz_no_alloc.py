"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (hosts that pass a library only its inputs and outputs, or that
forbid cudaMalloc). Its workspace is a fixed device array inside libfa. This
test calls it through the C ABI twice in a row and checks each result
element by element against the fp64 oracle (attn_bwd_ref) and against the
existing fa_bwd entry point given a caller-owned workspace, both within the
tolerance of the other GPU parity tests.

The file name makes pytest collect it after every other test file.
"""

import ctypes

import pytest
import torch

import oracle
from exact_io_aware_56_b200 import fa, make_inputs, to_f64

from .parity import assert_close_abs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20  # FA_BWD_NOALLOC_SCRATCH_BYTES in include/fa.h


def _noalloc():
    L = fa.lib()
    f = L.fa_bwd_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp] * 9 + [i, i, i, i, i, i, ctypes.c_float, vp]
    f.restype = i
    return f


def test_noalloc_matches_oracle_and_fa_bwd_twice():
    B, Hq, Hkv, N, d, causal = 1, 4, 2, 1000, 128, True
    assert fa.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) <= SCRATCH_BYTES
    scale = d ** -0.5
    host = make_inputs(B, Hq, Hkv, N, d, seed=2024)
    dev = {k: v.cuda() for k, v in host.items()}
    ref = {k: to_f64(v) for k, v in host.items()}
    want = oracle.attn_bwd_ref(ref["q"], ref["k"], ref["v"], ref["dout"], causal, scale)
    o, lse = fa.attention_forward(dev["q"], dev["k"], dev["v"], causal, scale)
    lib_out = fa.attention_backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, causal, scale)
    torch.cuda.synchronize()
    lib_out = [to_f64(t) for t in lib_out]
    f = _noalloc()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        dq, dk, dv = torch.empty_like(dev["q"]), torch.empty_like(dev["k"]), torch.empty_like(dev["v"])
        rc = f(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(), o.data_ptr(), dev["dout"].data_ptr(),
               lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, N, d, int(causal),
               scale, stream)
        assert rc == fa.FA_OK, fa.status_string(rc)
        torch.cuda.synchronize()
        assert fa.fa_check_device_error() == fa.FA_OK
        for name, got, w, lo in zip(("dQ", "dK", "dV"), (dq, dk, dv), want, lib_out):
            assert_close_abs(f"{name} vs oracle (call {call + 1})", to_f64(got), w)
            assert_close_abs(f"{name} vs fa_bwd (call {call + 1})", to_f64(got), lo)


def test_noalloc_rejects_shapes_beyond_its_array():
    f = _noalloc()
    p = ctypes.c_void_p(1 << 20)
    # 1 * 16 * 8192 rows of 128 fp32 values need 64 MiB > 32 MiB.
    rc = f(p, p, p, p, p, p, p, p, p, 1, 16, 16, 8192, 128, 1, 0.088, None)
    assert rc == fa.FA_ERR_UNSUPPORTED
    rc = f(p, p, p, p, p, p, p, p, p, 0, 1, 1, 16, 64, 0, 0.125, None)
    assert rc == fa.FA_ERR_INVALID_ARGUMENT
    rc = f(p, p, p, p, p, p, p, p, p, 1, 1, 1, 16, 96, 0, 0.125, None)
    assert rc == fa.FA_ERR_UNSUPPORTED
