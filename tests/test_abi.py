"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments before touching the device (no GPU needed)."""

import ctypes
import os
import re
import subprocess

import pytest

from exact_io_aware_56_b200 import fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(fa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(fa.LIB_PATH):
        from exact_io_aware_56_b200 import build
        build.build()
    return fa.lib()


def test_headers_declare_the_entry_points():
    names = declared_functions()
    for n in ["fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_status_string", "fa_check_device_error",
              "fa_set_watchdog_ns", "fa_test_set_fault"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", out, flags=re.M))
    for n in declared_functions():
        assert n in exported, n
        assert getattr(L, n) is not None


def test_status_strings(L):
    for s in range(5):
        assert len(fa.status_string(s)) > 0
    assert "unknown" in fa.status_string(99)


def test_invalid_arguments_rejected_before_launch(L):
    nul = None
    p = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: rejected before use
    mis = ctypes.c_void_p((1 << 20) + 8)
    ok_args = dict(B=1, Hq=2, Hkv=1, N=16, d=64, causal=0, scale=0.125)

    def fwd(q=p, k=p, v=p, o=p, lse=p, **kw):
        a = dict(ok_args, **kw)
        return L.fa_fwd(q, k, v, o, lse, a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["causal"], a["scale"], None)

    assert fwd(q=nul) == fa.FA_ERR_INVALID_ARGUMENT
    assert fwd(lse=nul) == fa.FA_ERR_INVALID_ARGUMENT
    assert fwd(k=mis) == fa.FA_ERR_INVALID_ARGUMENT
    assert fwd(N=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert fwd(B=-1) == fa.FA_ERR_INVALID_ARGUMENT
    assert fwd(causal=2) == fa.FA_ERR_INVALID_ARGUMENT
    assert fwd(scale=float("nan")) == fa.FA_ERR_INVALID_ARGUMENT
    assert fwd(scale=0.0) == fa.FA_ERR_INVALID_ARGUMENT
    assert fwd(scale=-1.0) == fa.FA_ERR_INVALID_ARGUMENT
    assert fwd(d=96) == fa.FA_ERR_UNSUPPORTED
    assert fwd(d=256) == fa.FA_ERR_UNSUPPORTED
    assert fwd(Hq=3, Hkv=2) == fa.FA_ERR_UNSUPPORTED

    def bwd(ws=p, ws_bytes=1 << 30, **kw):
        a = dict(ok_args, **kw)
        return L.fa_bwd(p, p, p, p, p, p, p, p, p, a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["causal"],
                        a["scale"], ws, ws_bytes, None)

    assert bwd(ws=nul) == fa.FA_ERR_INVALID_ARGUMENT
    assert bwd(ws_bytes=16) == fa.FA_ERR_INVALID_ARGUMENT
    assert bwd(d=32) == fa.FA_ERR_UNSUPPORTED


def test_workspace_size_formula(L):
    # fp32 D per query row plus an fp32 dQ accumulator per element, plus slack.
    B, Hq, Hkv, N, d = 2, 4, 2, 300, 128
    n = L.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d)
    assert n >= B * Hq * N * 4 + B * Hq * N * d * 4
    assert n < B * Hq * N * 4 + B * Hq * N * d * 4 + (1 << 20)
    assert L.fa_bwd_workspace_bytes(1, 1, 1, 16, 96) == 0
    assert L.fa_bwd_workspace_bytes(0, 1, 1, 16, 64) == 0


def test_other_entry_points_reject_bad_arguments_before_launch(L):
    p = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: rejected before use
    mis = ctypes.c_void_p((1 << 20) + 8)
    INV, UNS = fa.FA_ERR_INVALID_ARGUMENT, fa.FA_ERR_UNSUPPORTED

    # Masked forward / backward: window < -1 or prefix < 0 is invalid.
    def fwdm(q=p, window=-1, prefix=0, d=64):
        return L.fa_fwd_masked(q, p, p, p, None, p, 1, 2, 1, 16, d, window, prefix, 0.125, None)

    assert fwdm(window=-2) == INV and fwdm(prefix=-1) == INV and fwdm(q=None) == INV and fwdm(d=96) == UNS

    def bwdm(window=-1, prefix=0, ws_bytes=1 << 30):
        return L.fa_bwd_masked(p, p, p, p, None, p, p, p, p, p, 1, 2, 1, 16, 64, window, prefix, 0.125, p,
                               ws_bytes, None)

    assert bwdm(window=-5) == INV and bwdm(prefix=-3) == INV and bwdm(ws_bytes=8) == INV

    # FP8 quantizer and forward.
    def quant(x=p, scales=p, BH=2, N=16, d=64, per_head=0):
        return L.fa_quantize_fp8(x, p, scales, BH, N, d, per_head, None)

    assert quant(x=None) == INV and quant(x=mis) == INV and quant(scales=ctypes.c_void_p((1 << 20) + 2)) == INV
    assert quant(BH=0) == INV and quant(N=-1) == INV and quant(per_head=2) == INV and quant(d=96) == UNS

    def fwd8(sq=p, d=128, Hq=2, Hkv=1, scale=0.1):
        return L.fa_fwd_fp8(p, sq, p, p, p, p, p, p, 1, Hq, Hkv, 16, d, 1, scale, None)

    assert fwd8(sq=None) == INV and fwd8(sq=ctypes.c_void_p((1 << 20) + 1)) == INV
    assert fwd8(scale=float("inf")) == INV and fwd8(d=64) == UNS and fwd8(Hq=3, Hkv=2) == UNS

    # Decode.
    def dec(q=p, Nq=1, Nk=16, d=64, ws_bytes=1 << 30, Hq=2, Hkv=1):
        return L.fa_decode(q, p, p, p, p, 1, Hq, Hkv, Nq, Nk, d, 1, 0.125, p, ws_bytes, None)

    assert dec(q=None) == INV and dec(q=mis) == INV and dec(Nq=17) == INV and dec(Nk=0) == INV
    assert dec(d=96) == UNS and dec(Hq=3, Hkv=2) == UNS and dec(ws_bytes=8) == INV
    assert L.fa_decode_workspace_bytes(1, 2, 1, 17, 16, 64) == 0
    assert L.fa_decode_workspace_bytes(1, 2, 1, 1, 16, 96) == 0
    assert L.fa_decode_workspace_bytes(1, 2, 1, 1, 16, 64) > 0

    # No-allocation backward: shapes it cannot hold are rejected before any CUDA call.
    L.fa_bwd_noalloc.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 6 + [ctypes.c_float, ctypes.c_void_p]
    L.fa_bwd_noalloc.restype = ctypes.c_int

    def bwdn(B=1, N=16, d=64):
        return L.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, 2, 1, N, d, 1, 0.125, None)

    assert bwdn(B=0) == INV and bwdn(d=96) == UNS and bwdn(N=1 << 20) == UNS
