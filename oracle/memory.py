"""Byte and element counts of the attention tensors (test infrastructure only).

These restate the memory arithmetic that the pages print, so that a test can
check the worked numbers, and so that the long-context test can bound the
device memory a kernel may use:

* FlashAttention: IO-aware exact attention, "Attention moves a lot of bytes"
  paragraph (the N x N score matrix at a given N, heads and element size) and
  the "ONE 120K-TOKEN PREFILL REQUEST" diagram (naive scores per head; Q, K,
  V, O per head; one logsumexp float per row).
* Same page, "NAIVE ATTENTION vs FLASHATTENTION" diagram: the 128 x 128 score
  tile held in on-chip memory.
* Flash Attention: memory-efficient transformers, "The Standard Attention
  Bottleneck": the number of scores of one sequence.
"""

from __future__ import annotations


def score_count(n: int) -> int:
    """Number of query-key scores of one head: N * N."""
    return n * n


def naive_score_bytes(n: int, heads: int = 1, elem_bytes: int = 2) -> int:
    """Bytes of the materialised N x N score matrix for ``heads`` heads."""
    return score_count(n) * elem_bytes * heads


def flash_state_bytes(n: int, d: int, heads: int = 1, elem_bytes: int = 2) -> int:
    """Bytes of Q, K, V and O (four N x d tensors) for ``heads`` heads."""
    return 4 * n * d * elem_bytes * heads


def lse_bytes(n: int, heads: int = 1) -> int:
    """Bytes of the per-row logsumexp (one fp32 per query row)."""
    return 4 * n * heads


def tile_bytes(rows: int, cols: int, elem_bytes: int = 2) -> int:
    """Bytes of one score tile held on chip."""
    return rows * cols * elem_bytes
