"""Exact attention in float64 on the CPU: the definition, written out.

TEST INFRASTRUCTURE ONLY (see the package docstring). Nothing on the product
path may import this module.

Shapes follow the kernels' layout: ``q`` is ``[B, Hq, N, d]``, ``k`` and ``v``
are ``[B, Hkv, N, d]``, ``dout`` is like ``q``. All arrays are float64.

What is computed (FlashAttention: IO-aware exact attention, "NAIVE" box of the
"NAIVE ATTENTION vs FLASHATTENTION" diagram): S = scale * Q K^T, P =
softmax(S) row by row, O = P V. The "FLASH" box of the same diagram, and the
"Four ideas" list (item "Online softmax"), state that the tiled online form
reaches the same O exactly, and that one logsumexp per query row is kept for
the backward pass; that value is L_i = log sum_j exp(S_ij) (natural log).

Readings taken where the pages are silent (each is listed in the design
notes):

* The softmax scale multiplies Q K^T before the mask and the softmax.
* Causal masking hides key j from query i when j > i (queries and keys have
  the same length, so top-left and bottom-right alignment agree).
* Sliding-window and prefix-LM masks ("FlashAttention: IO-aware exact
  attention", "The honest limits": separate implementations, not a flag)
  are read as: key j is visible to query i iff (j <= i and i - j <= window)
  or j < prefix. window = None means no window (plain causal); prefix = 0
  means no prefix. Every row then sees at least its own key.
* Grouped-query attention (the "PREFILL PATH" diagram's notes on decode and
  the explainer's "Use with GQA") groups query heads contiguously: query head
  h reads KV head h // (Hq // Hkv).
* The FLASH box prints the loop body but not the last step; the plain reading
  is O <- O / l and L = m + ln l.
* The backward pass (the "Four ideas" item "Recomputation in the backward
  pass") is the textbook gradient of the definition: dV = P^T dO,
  dP = dO V^T, D_i = sum_j P_ij dP_ij, dS = P o (dP - D), dQ = scale dS K,
  dK = scale dS^T Q, summed over the query heads that share a KV head.
"""

from __future__ import annotations

import numpy as np

# Rows of S materialised at once by the blocked helpers. Only bounds memory;
# each row's arithmetic is unchanged by it.
_ROW_CHUNK = 512


def kv_head_of(hq: int, Hq: int, Hkv: int) -> int:
    """KV head read by query head ``hq``: contiguous groups of Hq/Hkv heads."""
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return hq // (Hq // Hkv)


def _check(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, Hq, N, d = q.shape
    if k.shape[0] != B or k.shape[2] != N or k.shape[3] != d or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, N, d] with q's B, N, d")
    if Hq % k.shape[1] != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return B, Hq, k.shape[1], N, d


def visible(row_ids, col_ids, causal, window=None, prefix=0):
    """Boolean [rows, cols] visibility of keys to queries (see module docstring)."""
    r = np.asarray(row_ids)[:, None]
    c = np.asarray(col_ids)[None, :]
    if not causal and window is None and prefix == 0:
        return np.ones((r.shape[0], c.shape[1]), dtype=bool)
    vis = c <= r
    if window is not None:
        vis &= (r - c) <= window
    if prefix:
        vis |= c < prefix
    return vis


def _masked(causal, window, prefix):
    return causal or window is not None or prefix > 0


def _scores(qrows, kmat, scale, causal, row_ids, window=None, prefix=0):
    """Rows of S = scale * Q K^T, with masked entries set to -inf.

    ``row_ids`` are the query positions of ``qrows`` (used by the masks).
    """
    S = scale * (qrows @ kmat.T)
    if _masked(causal, window, prefix):
        S[~visible(row_ids, np.arange(kmat.shape[0]), True, window, prefix)] = -np.inf
    return S


def _softmax_rows(S):
    """Two-pass softmax of each row (max, then normalised exponentials).

    Returns P and the row logsumexp L = m + ln(sum exp(S - m)).
    """
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    l = E.sum(axis=1, keepdims=True)
    return E / l, (m + np.log(l))[:, 0]


def attn_fwd_ref(q, k, v, causal: bool, scale: float, window=None, prefix=0):
    """Naive forward: S and P materialised, two-pass softmax, O = P V.

    FlashAttention: IO-aware exact attention, "NAIVE" box of the "NAIVE
    ATTENTION vs FLASHATTENTION" diagram (S = Q K^T, P = softmax(S),
    O = P V), plus the logsumexp of the "FLASH" box.

    Returns ``(O, L)`` with O like ``q`` and L ``[B, Hq, N]``.
    """
    B, Hq, Hkv, N, d = _check(q, k, v)
    O = np.empty_like(q, dtype=np.float64)
    L = np.empty((B, Hq, N), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            for r0 in range(0, N, _ROW_CHUNK):
                rows = np.arange(r0, min(N, r0 + _ROW_CHUNK))
                S = _scores(q[b, h, rows], k[b, g], scale, causal, rows, window, prefix)
                P, Lr = _softmax_rows(S)
                O[b, h, rows] = P @ v[b, g]
                L[b, h, rows] = Lr
    return O, L


def softmax_state(S, V):
    """Partial softmax state of one block of keys for each query row.

    For score rows ``S`` [rows, keys] (masked entries -inf) and the block's
    values ``V`` [keys, d] the state is (m, l, U): the row max m of S, the
    sum l of exp(S - m) and the unnormalised output U = exp(S - m) V. A row
    with every key of the block masked has m = -inf, l = 0 and U = 0 (the
    empty state). The normalised output of the block alone is U / l.
    """
    m = S.max(axis=1)
    ref = np.where(np.isneginf(m), 0.0, m)
    E = np.exp(S - ref[:, None])
    return m, E.sum(axis=1), E @ V


def merge_softmax_states(a, b):
    """Softmax state over the union of two disjoint key sets.

    FlashAttention: IO-aware exact attention, "Four ideas" list, item
    "Online softmax": a partial output is rescaled to a new, larger maximum
    and the rescale is exact; Flash Attention: memory-efficient
    transformers, "Online Softmax": the normalisation is updated per block
    instead of in a second pass. Written as the identity behind both: with
    M = max(m_a, m_b), sum_j exp(S_j - M) splits over the two key sets as
    e^(m_a - M) l_a + e^(m_b - M) l_b, and likewise for U. The operation
    is associative and commutative (up to rounding), so any order of
    merging gives the softmax over all keys. Empty states (m = -inf)
    contribute nothing.
    """
    ma, la, Ua = a
    mb, lb, Ub = b
    M = np.maximum(ma, mb)
    ref = np.where(np.isneginf(M), 0.0, M)
    fa = np.where(np.isneginf(ma), 0.0, np.exp(ma - ref))
    fb = np.where(np.isneginf(mb), 0.0, np.exp(mb - ref))
    return M, fa * la + fb * lb, fa[:, None] * Ua + fb[:, None] * Ub


def attn_fwd_online_ref(q, k, v, causal: bool, scale: float,
                        block_q: int = 128, block_k: int = 128, window=None, prefix=0, order=None):
    """Tiled forward built from per-block softmax states and their merge.

    Each (query block, key block) pair yields its own softmax state
    (:func:`softmax_state`); a query block's states over all key blocks are
    combined by :func:`merge_softmax_states`, so no N x N array is ever
    built and only (m, l, U) of a query block persist between key blocks
    (FlashAttention: IO-aware exact attention, "PREFILL PATH" diagram: only
    m, l and O stay on chip). The result is O = U / l and the row logsumexp
    L = m + ln l (natural log; the pages keep one logsumexp per query row).

    ``order`` (optional) is a permutation of the key-block indices giving the
    order in which states are merged, left to right; by default they are
    merged in ascending order, the order of a kernel streaming K/V blocks.
    Since the merge is associative and commutative, every order must give
    the two-pass result. Returns ``(O, L)`` like :func:`attn_fwd_ref`.
    """
    B, Hq, Hkv, N, d = _check(q, k, v)
    if block_q < 1 or block_k < 1:
        raise ValueError("block sizes must be positive")
    starts = list(range(0, N, block_k))
    if order is None:
        order = range(len(starts))
    elif sorted(order) != list(range(len(starts))):
        raise ValueError("order must be a permutation of the key-block indices")
    O_out = np.empty_like(q, dtype=np.float64)
    L_out = np.empty((B, Hq, N), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            for i0 in range(0, N, block_q):
                rows = np.arange(i0, min(N, i0 + block_q))
                state = (np.full(len(rows), -np.inf), np.zeros(len(rows)), np.zeros((len(rows), d)))
                for jb in order:
                    cols = np.arange(starts[jb], min(N, starts[jb] + block_k))
                    S = scale * (q[b, h, rows] @ k[b, g, cols].T)
                    if _masked(causal, window, prefix):
                        S[~visible(rows, cols, True, window, prefix)] = -np.inf
                    state = merge_softmax_states(state, softmax_state(S, v[b, g, cols]))
                m, l, U = state
                O_out[b, h, rows] = U / l[:, None]
                L_out[b, h, rows] = m + np.log(l)
    return O_out, L_out


def attn_bwd_ref(q, k, v, dout, causal: bool, scale: float, window=None, prefix=0):
    """Gradients of sum(dout * O) with respect to q, k, v.

    The pages state only that the backward pass rebuilds P from Q, K and L
    ("Four ideas", item "Recomputation in the backward pass"; blog section
    "Recomputation in the Backward Pass"). The formulas are the textbook
    gradient of softmax attention, materialised here row block by row block:
    P is rebuilt from S with the row logsumexp, dV = P^T dO, dP = dO V^T,
    D_i = sum_j P_ij dP_ij, dS = P o (dP - D), dQ = scale dS K and
    dK = scale dS^T Q. KV heads shared by several query heads sum the
    contributions of all of them.

    Returns ``(dq, dk, dv)`` shaped like ``q``, ``k``, ``v``.
    """
    B, Hq, Hkv, N, d = _check(q, k, v)
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros_like(k, dtype=np.float64)
    dv = np.zeros_like(v, dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            for r0 in range(0, N, _ROW_CHUNK):
                rows = np.arange(r0, min(N, r0 + _ROW_CHUNK))
                S = _scores(q[b, h, rows], k[b, g], scale, causal, rows, window, prefix)
                P, _ = _softmax_rows(S)
                dO = dout[b, h, rows]
                dv[b, g] += P.T @ dO
                dP = dO @ v[b, g].T
                D = (P * dP).sum(axis=1, keepdims=True)
                dS = P * (dP - D)
                dq[b, h, rows] = scale * (dS @ k[b, g])
                dk[b, g] += scale * (dS.T @ q[b, h, rows])
    return dq, dk, dv


def attn_fwd_rows(q, k, v, causal: bool, scale: float, b: int, h: int, rows, window=None, prefix=0):
    """O and L of query head ``h`` of batch ``b`` at the given query rows only.

    Same arithmetic as :func:`attn_fwd_ref` restricted to some rows (each row
    of the definition depends only on its own row of S). Returns
    ``(O_rows [len(rows), d], L_rows [len(rows)])``.
    """
    _, Hq, Hkv, _, _ = _check(q, k, v)
    g = kv_head_of(h, Hq, Hkv)
    rows = np.asarray(rows)
    O = np.empty((len(rows), q.shape[3]))
    L = np.empty(len(rows))
    for c0 in range(0, len(rows), _ROW_CHUNK):
        rr = rows[c0:c0 + _ROW_CHUNK]
        S = _scores(q[b, h, rr], k[b, g], scale, causal, rr, window, prefix)
        P, Lr = _softmax_rows(S)
        O[c0:c0 + len(rr)] = P @ v[b, g]
        L[c0:c0 + len(rr)] = Lr
    return O, L


def attn_bwd_rows(q, k, v, dout, causal: bool, scale: float, b: int, h: int, rows, window=None, prefix=0):
    """dQ of query head ``h`` of batch ``b`` at the given query rows only.

    dQ_i = scale * sum_j P_ij (dP_ij - D_i) K_j needs only row i of P and dP
    (D_i is a sum along that same row), so it is exact for a subset of rows.
    """
    _, Hq, Hkv, _, _ = _check(q, k, v)
    g = kv_head_of(h, Hq, Hkv)
    rows = np.asarray(rows)
    dq = np.empty((len(rows), q.shape[3]))
    for c0 in range(0, len(rows), _ROW_CHUNK):
        rr = rows[c0:c0 + _ROW_CHUNK]
        S = _scores(q[b, h, rr], k[b, g], scale, causal, rr, window, prefix)
        P, _ = _softmax_rows(S)
        dP = dout[b, h, rr] @ v[b, g].T
        D = (P * dP).sum(axis=1, keepdims=True)
        dq[c0:c0 + len(rr)] = scale * ((P * (dP - D)) @ k[b, g])
    return dq


def attn_bwd_kv_rows(q, k, v, dout, causal: bool, scale: float, b: int, g: int, keys, window=None, prefix=0):
    """dK and dV of KV head ``g`` of batch ``b`` at the given key rows only.

    Column j of P and dS depends on every query row's logsumexp and D_i, so
    all query rows of every query head sharing KV head ``g`` are rebuilt
    (row block by row block) and only the requested key columns are kept.
    Returns ``(dk_rows [len(keys), d], dv_rows [len(keys), d])``.
    """
    _, Hq, Hkv, N, d = _check(q, k, v)
    keys = np.asarray(keys)
    r = Hq // Hkv
    dk = np.zeros((len(keys), d))
    dv = np.zeros((len(keys), d))
    for h in range(g * r, (g + 1) * r):
        for r0 in range(0, N, _ROW_CHUNK):
            rows = np.arange(r0, min(N, r0 + _ROW_CHUNK))
            S = _scores(q[b, h, rows], k[b, g], scale, causal, rows, window, prefix)
            P, _ = _softmax_rows(S)
            dO = dout[b, h, rows]
            dP = dO @ v[b, g].T
            D = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dv += P[:, keys].T @ dO
            dk += scale * (dS[:, keys].T @ q[b, h, rows])
    return dk, dv


def attn_decode_ref(q, k, v, scale: float, causal: bool = True):
    """Decode / short-query attention: Nq new queries against an Nk-key cache.

    FlashAttention: IO-aware exact attention, "PREFILL PATH" diagram (after
    the prefill "decode loop starts (1 token at a time, now bound by
    KV-cache bandwidth ...)") and "Two notes" (decode reads the KV cache).
    The same definition as :func:`attn_fwd_ref` with ``q`` of shape
    [B, Hq, Nq, d] and ``k``, ``v`` of shape [B, Hkv, Nk, d], Nq <= Nk.
    Reading taken: the new queries are the last Nq positions of the
    sequence, so query i sits at position Nk - Nq + i and, when causal, sees
    keys j <= Nk - Nq + i (bottom-right alignment). Nq = 1 sees every key.
    Returns ``(O [B, Hq, Nq, d], L [B, Hq, Nq])``.
    """
    if q.ndim != 4 or k.ndim != 4 or v.shape != k.shape:
        raise ValueError("q must be [B, Hq, Nq, d]; k and v [B, Hkv, Nk, d]")
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != d or Hq % Hkv != 0 or Nq > Nk:
        raise ValueError("shapes do not match (need Nq <= Nk and Hq a multiple of Hkv)")
    O = np.empty((B, Hq, Nq, d))
    L = np.empty((B, Hq, Nq))
    pos = np.arange(Nk - Nq, Nk)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            S = _scores(q[b, h], k[b, g], scale, causal, pos)
            P, Lr = _softmax_rows(S)
            O[b, h] = P @ v[b, g]
            L[b, h] = Lr
    return O, L
