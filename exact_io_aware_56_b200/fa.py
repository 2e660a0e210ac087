"""ctypes binding of libfa.so (include/fa.h): argument marshalling only.

Each function takes torch CUDA tensors, checks that they have the layout the
C ABI documents, and passes raw device pointers, sizes and the current CUDA
stream to the library. All arithmetic happens in the CUDA kernels; there is
no CPU fallback, and a missing library or device raises ``RuntimeError``.
"""

from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa.so")

FA_OK = 0
FA_ERR_INVALID_ARGUMENT = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_CUDA = 3
FA_ERR_TIMEOUT = 4

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Loads libfa.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_io_aware_56_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    L.fa_fwd.restype = i
    L.fa_fwd_with_residual.argtypes = [vp] * 6 + [i, i, i, i, i, i, f, vp]
    L.fa_fwd_with_residual.restype = i
    L.fa_bwd_workspace_bytes.argtypes = [i, i, i, i, i]
    L.fa_bwd_workspace_bytes.restype = sz
    L.fa_bwd.argtypes = [vp] * 9 + [i, i, i, i, i, i, f, vp, sz, vp]
    L.fa_bwd.restype = i
    L.fa_bwd_with_residual.argtypes = [vp] * 10 + [i, i, i, i, i, i, f, vp, sz, vp]
    L.fa_bwd_with_residual.restype = i
    L.fa_fwd_masked.argtypes = [vp] * 6 + [i, i, i, i, i, i, i, f, vp]
    L.fa_fwd_masked.restype = i
    L.fa_bwd_masked.argtypes = [vp] * 10 + [i, i, i, i, i, i, i, f, vp, sz, vp]
    L.fa_bwd_masked.restype = i
    L.fa_quantize_fp8.argtypes = [vp, vp, vp, i, i, i, i, vp]
    L.fa_quantize_fp8.restype = i
    L.fa_fwd_fp8.argtypes = [vp] * 8 + [i, i, i, i, i, i, f, vp]
    L.fa_fwd_fp8.restype = i
    L.fa_decode_workspace_bytes.argtypes = [i, i, i, i, i, i]
    L.fa_decode_workspace_bytes.restype = sz
    L.fa_decode.argtypes = [vp] * 5 + [i, i, i, i, i, i, i, f, vp, sz, vp]
    L.fa_decode.restype = i
    L.fa_status_string.argtypes = [i]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_check_device_error.argtypes = [vp]
    L.fa_check_device_error.restype = i
    L.fa_set_watchdog_ns.argtypes = [ctypes.c_uint64]
    L.fa_set_watchdog_ns.restype = None
    L.fa_test_set_fault.argtypes = [i]
    L.fa_test_set_fault.restype = None
    L.fa_profile_set_bwd_events.argtypes = [vp, vp]
    L.fa_profile_set_bwd_events.restype = None
    L.fa_profile_set_decode_event.argtypes = [vp]
    L.fa_profile_set_decode_event.restype = None
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check_tensor(name, t, dtype, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise RuntimeError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.get_device() != torch.cuda.current_device():
        # The library launches on the current device with raw pointers.
        raise ValueError(f"{name} is on cuda:{t.get_device()} but the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _check_workspace(workspace):
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    if workspace.get_device() != torch.cuda.current_device():
        raise ValueError(f"workspace is on cuda:{workspace.get_device()} but the current device is "
                         f"cuda:{torch.cuda.current_device()}")


def _shapes(q, k):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, H, N, d]")
    B, Hq, N, d = q.shape
    return B, Hq, k.shape[1], N, d


def _mask_args(causal, window, prefix):
    if window is None and not prefix:
        return None
    if not causal:
        raise ValueError("window / prefix masks extend the causal mask: pass causal=True")
    return (-1 if window is None else int(window), int(prefix))


def fa_fwd(q, k, v, o, lse, causal: bool, scale: float, stream=None, o_resid=None, window=None,
           prefix: int = 0) -> None:
    """Forward pass into caller-owned ``o`` [B,Hq,N,d] bf16 and ``lse`` [B,Hq,N] fp32.

    With ``o_resid`` (bf16, like ``o``) this calls ``fa_fwd_with_residual``;
    with a ``window`` or a ``prefix`` (causal only) it calls ``fa_fwd_masked``.
    """
    B, Hq, Hkv, N, d = _shapes(q, k)
    bf = torch.bfloat16
    qa, ka, va, oa = (_check_tensor("q", q, bf, (B, Hq, N, d)), _check_tensor("k", k, bf, (B, Hkv, N, d)),
                      _check_tensor("v", v, bf, (B, Hkv, N, d)), _check_tensor("o", o, bf, (B, Hq, N, d)))
    la = _check_tensor("lse", lse, torch.float32, (B, Hq, N))
    mask = _mask_args(causal, window, prefix)
    tail = (B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream))
    if mask is not None:
        ra = None if o_resid is None else _check_tensor("o_resid", o_resid, bf, (B, Hq, N, d))
        rc, name = lib().fa_fwd_masked(qa, ka, va, oa, ra, la, B, Hq, Hkv, N, d, *mask, float(scale),
                                       _stream(stream)), "fa_fwd_masked"
    elif o_resid is None:
        rc, name = lib().fa_fwd(qa, ka, va, oa, la, *tail), "fa_fwd"
    else:
        ra = _check_tensor("o_resid", o_resid, bf, (B, Hq, N, d))
        rc, name = lib().fa_fwd_with_residual(qa, ka, va, oa, ra, la, *tail), "fa_fwd_with_residual"
    if rc != FA_OK:
        raise FaError(rc, name)


def fa_bwd_workspace_bytes(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_bytes(B, Hq, Hkv, N, d))


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, causal: bool, scale: float, workspace, stream=None,
           o_resid=None, window=None, prefix: int = 0) -> None:
    """Backward pass into caller-owned ``dq``, ``dk``, ``dv`` using ``workspace`` (uint8 CUDA tensor).

    With ``o_resid`` (from :func:`fa_fwd`) this calls ``fa_bwd_with_residual``.
    """
    B, Hq, Hkv, N, d = _shapes(q, k)
    bf = torch.bfloat16
    args = [_check_tensor("q", q, bf, (B, Hq, N, d)), _check_tensor("k", k, bf, (B, Hkv, N, d)),
            _check_tensor("v", v, bf, (B, Hkv, N, d)), _check_tensor("o", o, bf, (B, Hq, N, d)),
            _check_tensor("dout", dout, bf, (B, Hq, N, d)),
            _check_tensor("lse", lse, torch.float32, (B, Hq, N)),
            _check_tensor("dq", dq, bf, (B, Hq, N, d)), _check_tensor("dk", dk, bf, (B, Hkv, N, d)),
            _check_tensor("dv", dv, bf, (B, Hkv, N, d))]
    _check_workspace(workspace)
    ws_bytes = workspace.numel() * workspace.element_size()
    mask = _mask_args(causal, window, prefix)
    tail = (B, Hq, Hkv, N, d, int(bool(causal)), float(scale), workspace.data_ptr(), ws_bytes, _stream(stream))
    if mask is not None:
        ra = None if o_resid is None else _check_tensor("o_resid", o_resid, bf, (B, Hq, N, d))
        rc, name = lib().fa_bwd_masked(*args[:4], ra, *args[4:], B, Hq, Hkv, N, d, *mask, float(scale),
                                       workspace.data_ptr(), ws_bytes, _stream(stream)), "fa_bwd_masked"
    elif o_resid is None:
        rc, name = lib().fa_bwd(*args, *tail), "fa_bwd"
    else:
        ra = _check_tensor("o_resid", o_resid, bf, (B, Hq, N, d))
        rc, name = lib().fa_bwd_with_residual(*args[:4], ra, *args[4:], *tail), "fa_bwd_with_residual"
    if rc != FA_OK:
        raise FaError(rc, name)


def fa_quantize_fp8(x, codes, scales, per_head: bool, stream=None) -> None:
    """e4m3 block quantization of ``x`` [B, H, N, d] bf16 into ``codes``
    (uint8, like x) and ``scales`` (fp32: [B*H, ceil(N/128)] per 128-row
    block, or [B*H] per head)."""
    if x.dim() != 4:
        raise ValueError("x must be [B, H, N, d]")
    B, H, N, d = x.shape
    nb = (N + 127) // 128
    xa = _check_tensor("x", x, torch.bfloat16, (B, H, N, d))
    ca = _check_tensor("codes", codes, torch.uint8, (B, H, N, d))
    sa = _check_tensor("scales", scales, torch.float32, (B * H,) if per_head else (B * H, nb))
    rc = lib().fa_quantize_fp8(xa, ca, sa, B * H, N, d, int(bool(per_head)), _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_quantize_fp8")


def fa_fwd_fp8(q8, sq, k8, sk, v8, sv, o, lse, causal: bool, scale: float, stream=None) -> None:
    """FP8-mode forward (d = 128): e4m3 codes ``q8`` [B,Hq,N,d], ``k8``/``v8``
    [B,Hkv,N,d] (uint8) with block scales ``sq`` [B*Hq, nb], ``sk``
    [B*Hkv, nb], ``sv`` [B*Hkv]; writes ``o`` (bf16) and ``lse`` (fp32)."""
    B, Hq, Hkv, N, d = _shapes(q8, k8)
    nb = (N + 127) // 128
    u8, f32 = torch.uint8, torch.float32
    args = [_check_tensor("q8", q8, u8, (B, Hq, N, d)), _check_tensor("sq", sq, f32, (B * Hq, nb)),
            _check_tensor("k8", k8, u8, (B, Hkv, N, d)), _check_tensor("sk", sk, f32, (B * Hkv, nb)),
            _check_tensor("v8", v8, u8, (B, Hkv, N, d)), _check_tensor("sv", sv, f32, (B * Hkv,)),
            _check_tensor("o", o, torch.bfloat16, (B, Hq, N, d)), _check_tensor("lse", lse, f32, (B, Hq, N))]
    rc = lib().fa_fwd_fp8(*args, B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_fp8")


def fa_decode_workspace_bytes(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int) -> int:
    return int(lib().fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d))


def fa_decode(q, k, v, o, lse, causal: bool, scale: float, workspace, stream=None) -> None:
    """Decode attention: ``q``, ``o`` [B,Hq,Nq,d] bf16 against the cache ``k``, ``v``
    [B,Hkv,Nk,d] bf16 (Nq <= Nk, queries at the last Nq positions); ``lse``
    [B,Hq,Nq] fp32; ``workspace`` a uint8 CUDA tensor of at least
    :func:`fa_decode_workspace_bytes` bytes."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q must be [B, Hq, Nq, d] and k [B, Hkv, Nk, d]")
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    bf = torch.bfloat16
    args = [_check_tensor("q", q, bf, (B, Hq, Nq, d)), _check_tensor("k", k, bf, (B, Hkv, Nk, d)),
            _check_tensor("v", v, bf, (B, Hkv, Nk, d)), _check_tensor("o", o, bf, (B, Hq, Nq, d)),
            _check_tensor("lse", lse, torch.float32, (B, Hq, Nq))]
    _check_workspace(workspace)
    rc = lib().fa_decode(*args, B, Hq, Hkv, Nq, Nk, d, int(bool(causal)), float(scale), workspace.data_ptr(),
                         workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_decode")


def fa_check_device_error(stream=None) -> int:
    return int(lib().fa_check_device_error(_stream(stream)))


def fa_set_watchdog_ns(ns: int) -> None:
    lib().fa_set_watchdog_ns(int(ns))


def fa_test_set_fault(code: int) -> None:
    lib().fa_test_set_fault(int(code))


def fa_profile_set_bwd_events(after_pre=None, after_main=None) -> None:
    """Hands two torch.cuda.Event objects (or None) to the timing hook."""
    ptr = lambda e: None if e is None else e.cuda_event
    lib().fa_profile_set_bwd_events(ptr(after_pre), ptr(after_main))


def fa_profile_set_decode_event(after_main=None) -> None:
    """Hands a torch.cuda.Event (or None) to the decode timing hook."""
    lib().fa_profile_set_decode_event(None if after_main is None else after_main.cuda_event)


# ------------------------------------------------------------ conveniences

def attention_forward(q, k, v, causal: bool, scale: float | None = None, stream=None, residual: bool = False,
                      window=None, prefix: int = 0):
    """Allocates ``o`` and ``lse`` with torch and runs :func:`fa_fwd`.

    Returns ``(o, lse)``, or ``(o, lse, o_resid)`` when ``residual`` is true.
    """
    B, Hq, Hkv, N, d = _shapes(q, k)
    scale = d ** -0.5 if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    o_resid = torch.empty_like(q) if residual else None
    fa_fwd(q, k, v, o, lse, causal, scale, stream, o_resid=o_resid, window=window, prefix=prefix)
    return (o, lse, o_resid) if residual else (o, lse)


def attention_backward(q, k, v, o, dout, lse, causal: bool, scale: float | None = None, workspace=None,
                       stream=None, o_resid=None, window=None, prefix: int = 0):
    """Allocates ``dq``, ``dk``, ``dv`` (and the workspace if not given) and runs :func:`fa_bwd`."""
    B, Hq, Hkv, N, d = _shapes(q, k)
    scale = d ** -0.5 if scale is None else scale
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_bytes(B, Hq, Hkv, N, d), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, causal, scale, workspace, stream, o_resid=o_resid, window=window,
           prefix=prefix)
    return dq, dk, dv


def attention_decode(q, k, v, causal: bool = True, scale: float | None = None, workspace=None, stream=None):
    """Allocates ``o``, ``lse`` (and the workspace if not given) and runs :func:`fa_decode`.

    Returns ``(o, lse)``.
    """
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    scale = d ** -0.5 if scale is None else scale
    if workspace is None:
        workspace = torch.empty(max(16, fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d)), dtype=torch.uint8,
                                device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    fa_decode(q, k, v, o, lse, causal, scale, workspace, stream)
    return o, lse


def quantize_fp8(x, per_head: bool = False, stream=None):
    """Allocates and returns ``(codes, scales)`` for :func:`fa_quantize_fp8`."""
    B, H, N, d = x.shape
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    shape = (B * H,) if per_head else (B * H, (N + 127) // 128)
    scales = torch.empty(shape, dtype=torch.float32, device=x.device)
    fa_quantize_fp8(x, codes, scales, per_head, stream)
    return codes, scales


def attention_forward_fp8(q, k, v, causal: bool, scale: float | None = None, stream=None):
    """Quantizes bf16 ``q``, ``k`` (per 128-row block) and ``v`` (per head) and
    runs :func:`fa_fwd_fp8`. Returns ``(o, lse, (q8, sq, k8, sk, v8, sv))``."""
    B, Hq, Hkv, N, d = _shapes(q, k)
    scale = d ** -0.5 if scale is None else scale
    q8, sq = quantize_fp8(q, False, stream)
    k8, sk = quantize_fp8(k, False, stream)
    v8, sv = quantize_fp8(v, True, stream)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    fa_fwd_fp8(q8, sq, k8, sk, v8, sv, o, lse, causal, scale, stream)
    return o, lse, (q8, sq, k8, sk, v8, sv)
