"""Per-block INT8 quantisation of Q and K and the block-sparse attention on
the quantised scores, as the SpargeAttention notes describe the QK path
([P3] section 2.4: the QK product runs on SageAttention's per-block
quantisation with dequantisation scales; P and V stay in 16-bit).

TEST INFRASTRUCTURE ONLY (see the package header).

Readings where the notes are silent (they name the scheme, not its
arithmetic):
  * a block is ``rows`` consecutive tokens of one head (the query block for
    Q, the key block for K) over all d channels; its scale is
    absmax / 127 and every value is mapped to rint(x * (127 / absmax)) in
    float32 (round half to even), so the codes lie in [-127, 127]; a block
    of zeros has scale 0 and codes 0;
  * no smoothing of K (no mean subtraction) and no other transform;
  * scores are (q8 . k8) * scale_q * scale_k / sqrt(d): the exact integer
    dot product times the two scales, which equals the dot product of the
    dequantised rows; the softmax, the lambda test and P V are those of the
    16-bit path.

Pins (tests/test_oracle_quant.py): a hand-worked block (codes, scale,
round-half-even); the per-element error bound |x - x~| <= scale / 2; the
block-to-row mapping on a tensor whose rows grow in magnitude; the score
error bound sum_j |q_j| s_k / 2 + |k_j| s_q / 2 + s_q s_k / 4; the integer
product times the scales equals the dequantised product; a zero block.
"""

from __future__ import annotations

import numpy as np

from . import attention as A


def quantize_blocks(x, rows: int):
    """x [..., N, d] (float32 values) -> (codes int8 [..., N, d], scales
    float32 [..., ceil(N / rows)]), one scale per ``rows`` tokens."""
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


def dequantize(codes, scales, rows: int):
    """codes * scale of each row's block, in float64."""
    codes = np.asarray(codes, dtype=np.float64)
    n = codes.shape[-2]
    per_row = np.repeat(np.asarray(scales, dtype=np.float64), rows, axis=-1)[..., :n]
    return codes * per_row[..., None]


def block_sparse_attention_qk8_heads(q, k, v, kept, bq, bk, causal=False, lam=A.NEG_INF, scale=None,
                                     heads=None, qblocks=None, skip_override=None, band=1e-3):
    """``attention.block_sparse_attention_heads`` with Q quantised per query
    block (bq tokens) and K per key block (bk tokens); V unchanged."""
    q8, sq = quantize_blocks(q, bq)
    k8, sk = quantize_blocks(k, bk)
    return A.block_sparse_attention_heads(dequantize(q8, sq, bq), dequantize(k8, sk, bk), v, kept, bq, bk,
                                          causal, lam, scale, heads, qblocks, skip_override, band)
