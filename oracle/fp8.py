"""FP8 (e4m3) block quantization and attention on the dequantized tensors.

TEST INFRASTRUCTURE ONLY (see the package docstring). Nothing on the product
path may import this module.

What the pages fix: FlashAttention-3 adds "FP8 support with block scaling"
("FlashAttention: IO-aware exact attention", "The generations", the
FlashAttention-3 item), and FP8 mode changes rounding, so accuracy checks
stay mandatory ("The honest limits", last item). Nothing more is printed:
no number format, no block shape, no placement of the scales. Readings taken
(each listed in the design notes):

* The 8-bit format is e4m3 without infinities ("fn"): 1 sign bit, 4
  exponent bits with bias 7, 3 mantissa bits, subnormals below 2^-6, the
  codes 0x7F and 0xFF are NaN, and the largest finite magnitude is 448.
  Conversion rounds to nearest, ties to even, and saturates at +-448.
* A block is 128 consecutive rows of one (batch, head) for Q and K (the
  row-block of a 128 x d tile), and the whole (batch, head) for V. Its scale
  is s = amax / 448 (amax = largest |x| in the block; s = 1 when the block
  is all zero); the codes are e4m3(x * (448 / amax)). Both the reciprocal
  and the product are taken in fp32, the precision the quantizing kernel
  works in, so that the codes are a bit-exact target.
* The attention that FP8 mode computes is exact attention on the
  dequantized tensors x_hat = code * s: S = scale * Q_hat K_hat^T, then the
  softmax and O = P V_hat as in ``attention.attn_fwd_ref``. Everything the
  kernel rounds beyond that (P fed to the second product in e4m3) is kernel
  error, bounded in the tests from the arithmetic.
"""

from __future__ import annotations

import numpy as np

from .attention import attn_fwd_ref

E4M3_MAX = 448.0
BLOCK_ROWS = 128


def e4m3_decode(codes) -> np.ndarray:
    """Values of e4m3 codes (uint8 array) as float64, from the bit fields:
    exponent field 0 is subnormal (m / 8 * 2^-6), else (1 + m / 8) *
    2^(e - 7); exponent 15 with mantissa 7 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def _positive_grid():
    """All finite non-negative e4m3 values with their codes, ascending."""
    codes = np.arange(0x00, 0x7F, dtype=np.uint8)  # 0x7F is NaN
    return e4m3_decode(codes), codes


def e4m3_encode(x) -> np.ndarray:
    """Nearest e4m3 code of each float (ties to the even code, i.e. the one
    whose mantissa's last bit is 0), saturating at +-448. The sign bit is
    the sign of x, zeros included, as in IEEE format conversions (a negative
    value that rounds to zero gives 0x80). NaN is not accepted."""
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN has no rounding target")
    vals, codes = _positive_grid()
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(vals, a, side="left"), 0, len(vals) - 1)
    lo = np.clip(hi - 1, 0, len(vals) - 1)
    d_lo, d_hi = a - vals[lo], vals[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((codes[hi] & 1) == 0))
    idx = np.where(pick_hi, hi, lo)
    out = codes[idx].astype(np.uint8)
    return np.where(np.signbit(x), out | 0x80, out).astype(np.uint8)


def quantize_blocks(x, block_rows: int | None = BLOCK_ROWS):
    """Block quantization of ``x`` [..., N, d] (float64 values that are
    exact fp32 numbers, e.g. upcast bf16). Rows are cut into blocks of
    ``block_rows`` (None: one block per leading index, i.e. per head).
    Returns (codes uint8 like x, scales float32 [..., n_blocks])."""
    x = np.asarray(x, dtype=np.float64)
    lead, (N, d) = x.shape[:-2], x.shape[-2:]
    br = N if block_rows is None else block_rows
    nb = (N + br - 1) // br
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.ones(lead + (nb,), dtype=np.float32)
    for idx in np.ndindex(*lead):
        for b in range(nb):
            blk = x[idx][b * br:(b + 1) * br]
            amax = np.float32(np.abs(blk).max()) if blk.size else np.float32(0)
            if amax == 0:
                continue  # codes stay 0, scale stays 1
            inv = np.float32(E4M3_MAX) / amax                     # fp32, correctly rounded
            y = (blk.astype(np.float32) * inv).astype(np.float64)  # fp32 product
            codes[idx][b * br:(b + 1) * br] = e4m3_encode(y)
            scales[idx + (b,)] = amax / np.float32(E4M3_MAX)
    return codes, scales


def dequantize_blocks(codes, scales, block_rows: int | None = BLOCK_ROWS) -> np.ndarray:
    """x_hat = code * scale of its block, in float64."""
    v = e4m3_decode(codes)
    N = v.shape[-2]
    br = N if block_rows is None else block_rows
    s = np.repeat(np.asarray(scales, dtype=np.float64), br, axis=-1)[..., :N]
    return v * s[..., None]


def attn_fwd_fp8_ref(q8, sq, k8, sk, v8, sv, causal: bool, scale: float):
    """FP8-mode forward: exact attention (``attn_fwd_ref``) on Q, K
    dequantized per 128-row block and V dequantized per head. ``q8``
    [B, Hq, N, d], ``k8``/``v8`` [B, Hkv, N, d] uint8 codes; ``sq`` [B, Hq,
    nb], ``sk`` [B, Hkv, nb], ``sv`` [B, Hkv, 1] (or [B, Hkv]) fp32 scales.
    Returns (O, L) as ``attn_fwd_ref`` does."""
    sv = np.asarray(sv).reshape(np.asarray(v8).shape[:-2] + (1,))
    q = dequantize_blocks(q8, sq)
    k = dequantize_blocks(k8, sk)
    v = dequantize_blocks(v8, sv, None)
    return attn_fwd_ref(q, k, v, causal, scale)
