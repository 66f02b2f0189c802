"""Per-block 8-bit quantisation of Q and K and the block-sparse attention on
the quantised scores, as the SpargeAttention notes describe the QK path
([P3] section 2.4: the QK product runs on SageAttention's per-block
quantisation with dequantisation scales; P and V stay in 16-bit).  Two code
formats: INT8 (the notes' SageAttention) and FP8 E4M3.

TEST INFRASTRUCTURE ONLY (see the package header).

Readings where the notes are silent (they name the scheme, not its
arithmetic):
  * a block is ``rows`` consecutive tokens of one head (the query block for
    Q, the key block for K) over all d channels; its scale is
    absmax / 127 and every value is mapped to rint(x * (127 / absmax)) in
    float32 (round half to even), so the codes lie in [-127, 127]; a block
    of zeros has scale 0 and codes 0;
  * FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
    largest finite 448, subnormals down to 2^-9, no infinities): scale
    absmax / 448, code = the E4M3 value nearest to x * (448 / absmax) in
    float32, ties to even, magnitudes above 448 saturated to 448; the rounding
    is written here from that definition (``round_e4m3``);
  * no smoothing of K (no mean subtraction) and no other transform;
  * scores are (q8 . k8) * scale_q * scale_k / sqrt(d): the exact dot
    product of the codes (integers, or E4M3 values) times the two scales,
    which equals the dot product of the dequantised rows; the softmax, the
    lambda test and P V are those of the 16-bit path.

Pins (tests/test_oracle_quant.py): a hand-worked block (codes, scale,
round-half-even); the per-element error bound |x - x~| <= scale / 2 (INT8),
<= 2^-4 |x| or half the subnormal step (E4M3); the E4M3 value table (all 126
positive finite values from the format definition: every one a fixed point,
midpoints to even, saturation at 448, byte codes of hand-picked values); the
block-to-row mapping on a tensor whose rows grow in magnitude; the score
error bound sum_j |q_j| s_k / 2 + |k_j| s_q / 2 + s_q s_k / 4; the integer
product times the scales equals the dequantised product; a zero block.
"""

from __future__ import annotations

import numpy as np

from . import attention as A


E4M3_MAX = 448.0


def round_e4m3(x):
    """Nearest E4M3 value (ties to even), saturated to +-448, as float64."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)                      # a = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -6)               # binade exponent; subnormals share 2^-6's step
    step = np.ldexp(1.0, e - 3)              # 3 mantissa bits
    r = np.minimum(np.rint(a / step) * step, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_byte(v):
    """Byte code of E4M3 values (exactly representable, |v| <= 448)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    sign = np.signbit(v).astype(np.uint8) << 7
    _, ex = np.frexp(a)
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, ex - 1 + 7, 0)
    mant = np.where(normal, np.ldexp(a, -(ex - 1)) * 8 - 8, a / 2.0 ** -9)
    return (sign | (exp_field.astype(np.uint8) << 3) | np.rint(mant).astype(np.uint8)).astype(np.uint8)


def e4m3_value(b):
    """float64 value of E4M3 byte codes (no NaN codes expected)."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1 + m / 8.0) * np.ldexp(1.0, e - 7))
    return sign * mag


def quantize_blocks(x, rows: int, fmt: str = "int8"):
    """x [..., N, d] (float32 values) -> (codes [..., N, d], scales float32
    [..., ceil(N / rows)]), one scale per ``rows`` tokens.  fmt "int8":
    codes int8; fmt "e4m3": codes are E4M3 bytes (uint8)."""
    if fmt == "e4m3":
        return _quantize_blocks_e4m3(x, rows)
    x = np.asarray(x, dtype=np.float32)
    n = x.shape[-2]
    nblk = -(-n // rows)
    codes = np.zeros(x.shape, dtype=np.int8)
    scales = np.zeros(x.shape[:-2] + (nblk,), dtype=np.float32)
    for b in range(nblk):
        blk = x[..., b * rows:(b + 1) * rows, :]
        amax = np.abs(blk).max(axis=(-2, -1)).astype(np.float32)
        with np.errstate(divide="ignore"):
            inv = np.where(amax > 0, np.float32(127.0) / amax, np.float32(0.0)).astype(np.float32)
        scales[..., b] = np.where(amax > 0, amax / np.float32(127.0), np.float32(0.0))
        q = np.rint(blk * inv[..., None, None])                      # float32 product, half to even
        codes[..., b * rows:(b + 1) * rows, :] = np.clip(q, -127, 127).astype(np.int8)
    return codes, scales


def _quantize_blocks_e4m3(x, rows: int):
    x = np.asarray(x, dtype=np.float32)
    n = x.shape[-2]
    nblk = -(-n // rows)
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.zeros(x.shape[:-2] + (nblk,), dtype=np.float32)
    for b in range(nblk):
        blk = x[..., b * rows:(b + 1) * rows, :]
        amax = np.abs(blk).max(axis=(-2, -1)).astype(np.float32)
        with np.errstate(divide="ignore"):
            inv = np.where(amax > 0, np.float32(E4M3_MAX) / amax, np.float32(0.0)).astype(np.float32)
        scales[..., b] = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(0.0))
        y = blk * inv[..., None, None]                               # float32 product
        codes[..., b * rows:(b + 1) * rows, :] = e4m3_byte(round_e4m3(y))
    return codes, scales


def dequantize(codes, scales, rows: int, fmt: str = "int8"):
    """codes * scale of each row's block, in float64."""
    codes = e4m3_value(codes) if fmt == "e4m3" else np.asarray(codes, dtype=np.float64)
    n = codes.shape[-2]
    per_row = np.repeat(np.asarray(scales, dtype=np.float64), rows, axis=-1)[..., :n]
    return codes * per_row[..., None]


def block_sparse_attention_qk8_heads(q, k, v, kept, bq, bk, causal=False, lam=A.NEG_INF, scale=None,
                                     heads=None, qblocks=None, skip_override=None, band=1e-3, fmt="int8"):
    """``attention.block_sparse_attention_heads`` with Q quantised per query
    block (bq tokens) and K per key block (bk tokens) in ``fmt``; V
    unchanged."""
    q8, sq = quantize_blocks(q, bq, fmt)
    k8, sk = quantize_blocks(k, bk, fmt)
    return A.block_sparse_attention_heads(dequantize(q8, sq, bq, fmt), dequantize(k8, sk, bk, fmt), v, kept, bq,
                                          bk, causal, lam, scale, heads, qblocks, skip_override, band)
