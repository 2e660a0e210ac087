"""Host logic of the decode kernel's stream-K partition (CPU, no GPU): the
plan that fa_decode builds for a shape and a CTA count, read through the
fa_test_decode_plan hook, must cut the key tiles of all units into G
contiguous runs balanced to one tile, keep every run within MS units, give
each (run, unit) pair its own partial slot, and fit the workspace that
fa_decode_workspace_bytes asks the caller for."""

import bisect
import ctypes
import itertools

import numpy as np
import pytest

from exact_io_aware_56_b200 import fa


def plan(B, Hq, Hkv, Nq, Nk, d, ctas):
    L = fa.lib()
    L.fa_test_decode_plan.argtypes = [ctypes.c_int] * 7 + [ctypes.POINTER(ctypes.c_longlong)]
    L.fa_test_decode_plan.restype = ctypes.c_int
    out = (ctypes.c_longlong * 8)()
    rc = L.fa_test_decode_plan(B, Hq, Hkv, Nq, Nk, d, ctas, out)
    return rc, dict(zip(["W", "T", "G", "MS", "R", "rho", "rv", "n_chunks"], list(out)))


def workspace_bytes(B, Hq, Hkv, Nq, Nk, d):
    L = fa.lib()
    L.fa_decode_workspace_bytes.argtypes = [ctypes.c_int] * 6
    L.fa_decode_workspace_bytes.restype = ctypes.c_size_t
    return L.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d)


def shapes():
    rng = np.random.default_rng(5)
    fixed = [(16, 32, 8, 1, 8192, 128), (4, 64, 8, 4, 32768, 128), (64, 16, 16, 1, 2048, 64),
             (1, 1, 1, 1, 1, 64), (1, 8, 1, 16, 128, 128), (3, 40, 2, 7, 129, 64), (2, 128, 1, 3, 1000, 128)]
    rand = []
    for _ in range(40):
        hkv = int(rng.choice([1, 2, 4, 8, 16]))
        ratio = int(rng.choice([1, 2, 4, 8, 16]))
        nk = int(rng.integers(1, 20000))
        nq = int(min(nk, rng.choice([1, 2, 3, 4, 7, 16, 33, 130])))
        rand.append((int(rng.integers(1, 70)), hkv * ratio, hkv, nq, nk, int(rng.choice([64, 128]))))
    return fixed + rand


@pytest.mark.parametrize("shape,ctas", list(itertools.product(shapes(), [1, 7, 148, 256, 1000])))
def test_decode_plan_invariants(shape, ctas):
    B, Hq, Hkv, Nq, Nk, d = shape
    rc, p = plan(B, Hq, Hkv, Nq, Nk, d, ctas)
    assert rc == fa.FA_OK
    W, T, G, MS = p["W"], p["T"], p["G"], p["MS"]
    # Units: (batch, KV head, chunk of 128 / rho rows); rows of one KV head are
    # replicated rho times over the 128 tensor-memory lanes.
    R = (Hq // Hkv) * Nq
    assert p["R"] == R and p["rho"] in (1, 2, 4) and R <= 128 // p["rho"] * p["n_chunks"]
    assert p["rv"] == min(R, 128 // p["rho"]) and (p["rho"] == 1 or R <= 128 // p["rho"])
    assert T == -(-Nk // 128) and W == B * Hkv * p["n_chunks"] * T
    assert 1 <= G <= min(ctas, 256, W)
    # Runs [lo(c), lo(c+1)) tile [0, W) in order, balanced to one tile.
    lo = [c * W // G for c in range(G + 1)]
    assert lo[0] == 0 and lo[-1] == W
    lens = np.diff(lo)
    assert lens.min() >= W // G and lens.max() <= -(-W // G)
    # The closed-form owner of a tile (used by the merge) agrees with a search.
    for t in sorted({0, W - 1, W // 2, *np.random.default_rng(W).integers(0, W, 64).tolist()}):
        owner = ((t + 1) * G + W - 1) // W - 1
        assert owner == bisect.bisect_right(lo, t) - 1
    # Every run touches at most MS units, so slot c * MS + (u - lo(c) // T)
    # is private to the pair (run c, unit u) and below G * MS.
    for c in range(G):
        if lo[c + 1] > lo[c]:
            first, last = lo[c] // T, (lo[c + 1] - 1) // T
            assert last - first + 1 <= MS
    # The partials fit the workspace the API asks for.
    need = G * MS * p["rho"] * p["rv"] * (d + 1) * 4
    assert need <= workspace_bytes(B, Hq, Hkv, Nq, Nk, d)


def test_decode_plan_rejects_what_fa_decode_rejects():
    out_rc = [plan(1, 3, 2, 1, 10, 128, 148)[0],   # Hq not a multiple of Hkv
              plan(1, 2, 2, 5, 4, 128, 148)[0],    # Nq > Nk
              plan(1, 2, 2, 1, 4, 96, 148)[0],     # d not 64 or 128
              plan(1, 2, 2, 1, 4, 128, 0)[0]]      # no CTAs
    assert out_rc == [fa.FA_ERR_UNSUPPORTED, fa.FA_ERR_INVALID_ARGUMENT, fa.FA_ERR_UNSUPPORTED,
                      fa.FA_ERR_INVALID_ARGUMENT]
