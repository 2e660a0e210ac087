"""GPU parity of the decode / short-query path (fa_decode) against the fp64
oracle's decode reference: one to a few queries per head against a cache,
GQA ratios 1-16, row chunks of every replication (<= 32, <= 64, > 64 and
> 128 rows per KV head), ragged cache lengths, both head dims, causal and
not, the serving-size workloads, exactness on saturated rows, determinism,
untouched guard bytes, and argument errors."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_56_b200 import DECODE_WORKLOADS, fa, make_decode_inputs, to_f64

from .parity import assert_close_abs, assert_close_lse

pytestmark = pytest.mark.gpu


def run_decode(host, causal, scale, ws_fill=None):
    dev = {k: t.cuda() for k, t in host.items()}
    B, Hq, Nq, d = dev["q"].shape
    Hkv, Nk = dev["k"].shape[1], dev["k"].shape[2]
    ws = torch.empty(max(16, fa.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d)), dtype=torch.uint8,
                     device="cuda")
    if ws_fill is not None:
        ws.fill_(ws_fill)
    o, lse = fa.attention_decode(dev["q"], dev["k"], dev["v"], causal, scale, workspace=ws)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == fa.FA_OK
    return o, lse


def check_decode(B, Hq, Hkv, Nq, Nk, d, causal, seed):
    host = make_decode_inputs(B, Hq, Hkv, Nq, Nk, d, seed)
    scale = d ** -0.5
    o, lse = run_decode(host, causal, scale)
    ref = {k: to_f64(t) for k, t in host.items()}
    O, L = oracle.attn_decode_ref(ref["q"], ref["k"], ref["v"], scale, causal)
    assert_close_abs("O", to_f64(o), O)
    assert_close_lse(to_f64(lse), L)


SHAPES = [  # (B, Hq, Hkv, Nq, Nk)
    (1, 1, 1, 1, 1), (2, 4, 1, 1, 300), (1, 8, 2, 3, 129), (1, 8, 1, 9, 1000), (2, 8, 1, 20, 600),
    (1, 2, 1, 70, 200), (3, 4, 2, 2, 130), (1, 16, 1, 5, 2000), (1, 1, 1, 33, 40), (1, 32, 32, 1, 4097),
    (2, 16, 1, 1, 128), (1, 4, 4, 128, 128),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("d", [64, 128])
def test_decode_shapes_causal(shape, d):
    check_decode(*shape, d, True, seed=500 + sum(shape) + d)


@pytest.mark.parametrize("shape", [(1, 4, 4, 5, 257), (2, 8, 2, 16, 700), (1, 2, 1, 100, 333)])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_shapes_noncausal(shape, d):
    check_decode(*shape, d, False, seed=600 + sum(shape) + d)


@pytest.mark.parametrize("name", sorted(DECODE_WORKLOADS))
def test_decode_workloads_full(name):
    w = DECODE_WORKLOADS[name]
    host = make_decode_inputs(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.seed)
    o, lse = run_decode(host, w.causal, w.scale)
    # The oracle on every (batch, KV head) of a seeded sample of 4 batches.
    rng = np.random.default_rng(w.seed + 1000)
    for b in np.sort(rng.choice(w.B, size=min(4, w.B), replace=False)):
        ref = {k: to_f64(t[b:b + 1]) for k, t in host.items()}
        O, L = oracle.attn_decode_ref(ref["q"], ref["k"], ref["v"], w.scale, w.causal)
        assert_close_abs("O", to_f64(o[b:b + 1]), O)
        assert_close_lse(to_f64(lse[b:b + 1]), L)


def test_decode_deterministic_and_workspace_independent():
    host = make_decode_inputs(2, 16, 2, 3, 3000, 128, 77)
    a = run_decode(host, True, 0.1, ws_fill=0)
    b = run_decode(host, True, 0.1, ws_fill=0xFF)  # NaN bit patterns in the workspace
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_decode_saturated_rows_exact():
    # Each query row's score on one chosen key exceeds all others by far more
    # than the fp32 underflow gap, so O = V[key] bit for bit and L is closed form.
    B, Hq, Hkv, Nq, Nk, d = 2, 8, 2, 3, 1000, 64
    alpha = 64.0
    g = torch.Generator().manual_seed(31)
    k = (torch.randint(0, 2, (B, Hkv, Nk, d), generator=g) * 2 - 1).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Nk, d, generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(31)
    pick = np.zeros((B, Hq, Nq), dtype=np.int64)
    q = torch.empty(B, Hq, Nq, d, dtype=torch.bfloat16)
    r = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            for i in range(Nq):
                pick[b, h, i] = rng.integers(0, Nk - Nq + i + 1)
                q[b, h, i] = (alpha * k[b, h // r, pick[b, h, i]].float()).to(torch.bfloat16)
    kf = k.double().numpy()
    scale = d ** -0.5
    for b in range(B):
        for h in range(Hq):
            kk = kf[b, h // r]
            for i in range(Nq):
                dots = kk @ kk[pick[b, h, i]]
                dots[pick[b, h, i]] = -np.inf
                dots[Nk - Nq + i + 1:] = -np.inf
                assert alpha * scale * np.log2(np.e) * (d - dots.max()) > 160.0
    o, lse = run_decode({"q": q, "k": k, "v": v}, True, scale)
    o = o.cpu()
    for b in range(B):
        for h in range(Hq):
            want = v[b, h // r, torch.from_numpy(pick[b, h])]
            assert torch.equal(o[b, h], want), (b, h)
    rel = (lse.cpu().double() / (scale * alpha * d) - 1.0).abs().max().item()
    assert rel < 2e-6, rel


def test_decode_guard_bytes_untouched():
    B, Hq, Hkv, Nq, Nk, d = 1, 8, 2, 2, 513, 128
    host = make_decode_inputs(B, Hq, Hkv, Nq, Nk, d, 5)
    dev = {k: t.cuda() for k, t in host.items()}
    n_o, n_l, pad = B * Hq * Nq * d, B * Hq * Nq, 4096
    obuf = torch.full((n_o + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((n_l + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    o = obuf[pad:pad + n_o].view(B, Hq, Nq, d)
    lse = lbuf[pad:pad + n_l].view(B, Hq, Nq)
    ws = torch.empty(fa.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d), dtype=torch.uint8, device="cuda")
    fa.fa_decode(dev["q"], dev["k"], dev["v"], o, lse, True, 0.09, ws)
    torch.cuda.synchronize()
    for buf, n in ((obuf, n_o), (lbuf, n_l)):
        assert (buf[:pad] == 7.0).all() and (buf[pad + n:] == 7.0).all()


def test_decode_argument_errors():
    host = make_decode_inputs(1, 4, 2, 2, 64, 64, 1)
    dev = {k: t.cuda() for k, t in host.items()}
    o = torch.empty_like(dev["q"])
    lse = torch.empty(1, 4, 2, dtype=torch.float32, device="cuda")
    need = fa.fa_decode_workspace_bytes(1, 4, 2, 2, 64, 64)
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FaError):
        fa.fa_decode(dev["q"], dev["k"], dev["v"], o, lse, True, 0.125, small)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FaError):
        fa.fa_decode(dev["q"], dev["k"], dev["v"], o, lse, True, float("nan"), ws)
    # More queries than cached keys.
    q = torch.zeros(1, 4, 65, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError):
        fa.fa_decode(q, dev["k"], dev["v"], torch.empty_like(q), torch.empty(1, 4, 65, device="cuda"), True,
                     0.125, torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
