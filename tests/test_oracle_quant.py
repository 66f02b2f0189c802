"""Pins of the per-block INT8 quantisation oracle (oracle.quant) against hand
arithmetic and closed-form bounds (CPU only)."""

import numpy as np
import pytest

from oracle import attention as A
from oracle import quant as Q


def test_hand_worked_block():
    """absmax 2: 127 / 2 = 63.5; 1 -> 63.5 -> 64 (half to even), -2 -> -127,
    0.5 -> 31.75 -> 32, 0 -> 0; 0.75 -> 47.625 -> 48; scale 2 / 127."""
    x = np.array([[[1.0, -2.0, 0.5, 0.0], [0.75, 0.0, 0.0, 0.0]]], dtype=np.float32)
    codes, scales = Q.quantize_blocks(x, 2)
    assert codes.tolist() == [[[64, -127, 32, 0], [48, 0, 0, 0]]]
    assert scales.tolist() == [np.float32(2.0) / np.float32(127.0)]
    # 1.5 * 127 / 3 = 63.5 exactly in float32 as well: half to even gives 64, 2.5 * (127/5) = 63.5 -> 64
    y = np.array([[[3.0, 1.5]], [[5.0, 2.5]]], dtype=np.float32)
    c2, _ = Q.quantize_blocks(y, 1)
    assert c2[..., 1].ravel().tolist() == [64, 64]


def test_half_to_even_both_ways():
    """x * 127 / absmax landing on k + 1/2 rounds to the even neighbour."""
    amax = np.float32(127.0)                       # inv = 1: codes are rint(x)
    x = np.array([[[amax, 0.5, 1.5, 2.5, -0.5, -1.5]]], dtype=np.float32)
    codes, scales = Q.quantize_blocks(x, 1)
    assert codes.ravel().tolist() == [127, 0, 2, 2, 0, -2]
    assert scales.ravel().tolist() == [1.0]


@pytest.mark.parametrize("rows", [1, 3, 64])
def test_error_bound_and_code_range(rows):
    rng = np.random.default_rng(rows)
    x = (rng.standard_normal((2, 3, 150, 16)) * rng.uniform(0.1, 10, size=(2, 3, 150, 1))).astype(np.float32)
    codes, scales = Q.quantize_blocks(x, rows)
    assert codes.min() >= -127 and codes.max() <= 127
    err = np.abs(Q.dequantize(codes, scales, rows) - x)
    bound = np.repeat(scales.astype(np.float64), rows, axis=-1)[..., :150, None] / 2
    assert np.all(err <= bound * (1 + 1e-6))
    # every block uses the full range: its absmax element maps to +-127
    for b in range(-(-150 // rows)):
        assert np.all(np.abs(codes[..., b * rows:(b + 1) * rows, :]).max(axis=(-2, -1)) == 127)


def test_block_to_row_mapping():
    """Rows whose magnitude is their index: block b's scale is the largest
    row index it holds, / 127."""
    n, rows = 10, 4
    x = np.repeat(np.arange(1, n + 1, dtype=np.float32)[:, None], 3, axis=1)[None]
    _, scales = Q.quantize_blocks(x, rows)
    assert scales.ravel().tolist() == pytest.approx([4 / 127, 8 / 127, 10 / 127], rel=1e-7)


def test_zero_block():
    x = np.zeros((1, 5, 4), dtype=np.float32)
    x[0, 4, 0] = 3.0
    codes, scales = Q.quantize_blocks(x, 4)
    assert not codes[0, :4].any() and scales[0, 0] == 0.0
    assert codes[0, 4, 0] == 127 and scales[0, 1] == np.float32(3.0) / np.float32(127.0)


def test_integer_product_and_score_bound():
    """(q8 . k8) * sq * sk is the dequantised dot product, and its distance
    to q . k is within sum_j |q_j| sk/2 + |k_j| sq/2 + sq sk/4."""
    rng = np.random.default_rng(8)
    q = rng.standard_normal((256, 128)).astype(np.float32)
    k = (rng.standard_normal((256, 128)) * 3).astype(np.float32)
    q8, sq = Q.quantize_blocks(q, 128)
    k8, sk = Q.quantize_blocks(k, 64)
    s_int = q8.astype(np.int64) @ k8.astype(np.int64).T
    sq_row = np.repeat(sq.astype(np.float64), 128)[:, None]
    sk_col = np.repeat(sk.astype(np.float64), 64)[None, :]
    s_deq = Q.dequantize(q8, sq, 128) @ Q.dequantize(k8, sk, 64).T
    assert np.allclose(s_int * sq_row * sk_col, s_deq, rtol=1e-12, atol=1e-12)
    s = q.astype(np.float64) @ k.astype(np.float64).T
    bound = (np.abs(q).sum(1)[:, None] * sk_col / 2 + np.abs(k).sum(1)[None, :] * sq_row / 2
             + 128 * sq_row * sk_col / 4)
    assert np.all(np.abs(s_deq - s) <= bound)


def test_quantised_attention_is_close_to_exact():
    """On N(0,1) inputs the quantised path stays close to the 16-bit
    definition: mean error about 1e-3, max about 1e-2 (a sanity pin on the
    scale placement: swapping the key blocks' scales gives mean 2e-2, max 0.4)."""
    rng = np.random.default_rng(2)
    n = 200
    q, k, v = (rng.standard_normal((1, 1, n, 128)).astype(np.float32) for _ in range(3))
    kept = np.ones((1, 1, 2, 4), dtype=bool)
    r8 = Q.block_sparse_attention_qk8_heads(q, k, v, kept, 128, 64)
    r = A.block_sparse_attention_heads(q, k, v, kept, 128, 64)
    d = np.abs(r8["out"] - r["out"])
    assert d.max() < 3e-2 and d.mean() < 3e-3
    assert np.max(np.abs(r8["lse"] - r["lse"])) < 3e-2
