"""Closed-form GPU checks on saturated attention: every query row has one
visible key whose score exceeds all its other visible scores by so much that
their weights underflow to exactly 0 in fp32. Softmax is then one-hot, so
exactly (the "FLASH" box of the "NAIVE ATTENTION vs FLASHATTENTION" diagram
on the page FlashAttention: IO-aware exact attention computes softmax(QK^T)V
and its logsumexp):

  O[r] = V[pi(r)]             bit for bit (bf16 in, bf16 out, weight 1.0)
  L[r] = scale * q_r . k_pi(r) up to fp32 rounding
  dV[j] = sum of dO[r] over the rows with pi(r) = j,  dQ = dK = 0

A row max that is not the exact maximum of the visible scores leaves the
dominant weight at 2^x with x != 0, whose bf16 rounding moves O by an ulp;
these checks see that where the tolerance of the random-input parity tests
does not.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_56_b200 import fa

pytestmark = pytest.mark.gpu

ALPHA = 64.0            # query = ALPHA * its chosen key (exact in bf16)
UNDERFLOW_LOG2 = 160.0  # gap in log2 units past which fp32 exp2 flushes to 0


def saturated_inputs(B, Hq, Hkv, N, d, causal, window, prefix, seed):
    """K rows of +-1, Q[r] = ALPHA * K[pi(r)] for a visible key pi(r); V and
    dO standard normal in bf16. Returns host tensors and pi."""
    g = torch.Generator().manual_seed(seed)
    k = (torch.randint(0, 2, (B, Hkv, N, d), generator=g) * 2 - 1).to(torch.bfloat16)
    v = torch.randn(B, Hkv, N, d, generator=g).to(torch.bfloat16)
    dout = torch.randn(B, Hq, N, d, generator=g).to(torch.bfloat16)
    rows = np.arange(N)
    pi = np.zeros((B, Hq, N), dtype=np.int64)
    vis = oracle.visible(rows, rows, causal, window, prefix) if causal else np.ones((N, N), dtype=bool)
    rng = np.random.default_rng(seed)
    for r in range(N):
        cand = np.nonzero(vis[r])[0]
        pi[:, :, r] = rng.choice(cand, size=(B, Hq))
    grp = Hq // Hkv
    q = torch.empty(B, Hq, N, d, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(Hq):
            q[b, h] = (ALPHA * k[b, h // grp, torch.from_numpy(pi[b, h])].float()).to(torch.bfloat16)
    # Precondition: every other visible score is below the chosen one by more
    # than the underflow gap (after scale * log2 e).
    scale = d ** -0.5
    kf = k.double().numpy()
    for b in range(B):
        for h in range(Hq):
            kk = kf[b, h // grp]
            dots = kk[pi[b, h]] @ kk.T
            dots[rows, pi[b, h]] = -np.inf
            dots[~vis] = -np.inf
            gap = d - dots.max(axis=1)
            assert (ALPHA * scale * np.log2(np.e) * gap[np.isfinite(gap)] > UNDERFLOW_LOG2).all()
    return {"q": q, "k": k, "v": v, "dout": dout}, pi


CASES = [  # (causal, window, prefix)
    (False, None, 0), (True, None, 0), (True, 0, 0), (True, 5, 0), (True, 200, 0), (True, None, 100),
    (True, 64, 150),
]


@pytest.mark.parametrize("causal,window,prefix", CASES)
@pytest.mark.parametrize("d", [64, 128])
def test_saturated_rows_exact(causal, window, prefix, d):
    B, Hq, Hkv, N = 1, 4, 2, 777
    host, pi = saturated_inputs(B, Hq, Hkv, N, d, causal, window, prefix, seed=900 + d + (window or 0) + prefix)
    dev = {k: t.cuda() for k, t in host.items()}
    scale = d ** -0.5
    kw = {} if not causal else {"window": window, "prefix": prefix}
    o, lse, res = fa.attention_forward(dev["q"], dev["k"], dev["v"], causal, scale, residual=True, **kw)
    dq, dk, dv = fa.attention_backward(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, causal, scale,
                                       o_resid=res, **kw)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error() == fa.FA_OK
    grp = Hq // Hkv
    o = o.cpu()
    for h in range(Hq):
        want = host["v"][0, h // grp, torch.from_numpy(pi[0, h])]
        bad = (o[0, h] != want).any(dim=1).nonzero().flatten().tolist()
        assert not bad, f"head {h}: O rows differ from V[pi(r)] at rows {bad[:10]} ({len(bad)} rows)"
    # q_r . k_pi(r) = ALPHA * (k . k) = ALPHA * d for +-1 keys.
    lse_want = scale * ALPHA * d * torch.ones(B, Hq, N, dtype=torch.float64)
    rel = ((lse.cpu().double() - lse_want).abs() / lse_want.abs()).max().item()
    assert rel < 2e-6, rel
    assert dq.abs().max().item() < 1e-3 and dk.abs().max().item() < 1e-3
    dv_want = torch.zeros(B, Hkv, N, d, dtype=torch.float64)
    for h in range(Hq):
        dv_want[0, h // grp].index_add_(0, torch.from_numpy(pi[0, h]), host["dout"][0, h].double())
    err = (dv.cpu().double() - dv_want).abs() - 2.0 ** -8 * dv_want.abs()
    assert err.max().item() <= 1e-6, err.max().item()
