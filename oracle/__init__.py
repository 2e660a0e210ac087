"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. This package is the independent definition that the
CUDA kernels are checked against. Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline / reference legs of ``bench.py`` may
import it. The product path (the ``exact_io_aware_56_b200`` package and its
CUDA library) never imports, links or calls anything here, and nothing here
imports the product package: the two share no code.

Every function is plain numpy in float64 and cites the passage of the source
pages it follows. Page titles used in citations:

* "FlashAttention: IO-aware exact attention" (mlapandio.dev daily term),
  its diagrams "NAIVE ATTENTION vs FLASHATTENTION" (boxes NAIVE and FLASH),
  "ONE 120K-TOKEN PREFILL REQUEST" and "PREFILL PATH", and its lists
  "Four ideas" and "The honest limits".
* "Flash Attention: memory-efficient transformers" (techtrendtracker blog),
  sections "The Standard Attention Bottleneck", "Recomputation in the
  Backward Pass" and "Online Softmax".

Parity status: every function here is pinned by a CPU test against closed
forms, identities, brute force or finite differences (tests/test_oracle_*.py);
none is "parity unpinned".
"""

from .attention import (  # noqa: F401
    attn_fwd_ref,
    attn_fwd_online_ref,
    merge_softmax_states,
    softmax_state,
    attn_bwd_ref,
    attn_fwd_rows,
    attn_bwd_rows,
    attn_bwd_kv_rows,
    attn_decode_ref,
    visible,
    kv_head_of,
)
from .fp8 import (  # noqa: F401
    attn_fwd_fp8_ref,
    dequantize_blocks,
    e4m3_decode,
    e4m3_encode,
    quantize_blocks,
)
from .memory import (  # noqa: F401
    naive_score_bytes,
    flash_state_bytes,
    lse_bytes,
    score_count,
    tile_bytes,
)
