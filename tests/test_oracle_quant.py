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


# --------------------------------------------------------------------------
# FP8 E4M3
# --------------------------------------------------------------------------

def _e4m3_table():
    """Every positive finite E4M3 value from the format definition."""
    vals = [m * 2.0 ** -9 for m in range(1, 8)]                       # subnormals
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue                                              # the NaN code
            vals.append((1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals)


def test_e4m3_table_is_fixed_and_byte_codes_round_trip():
    t = _e4m3_table()
    assert t.size == 126 and t.max() == 448.0 and t.min() == 2.0 ** -9
    assert np.array_equal(Q.round_e4m3(t), t) and np.array_equal(Q.round_e4m3(-t), -t)
    codes = Q.e4m3_byte(np.concatenate([t, -t, [0.0]]))
    assert np.array_equal(Q.e4m3_value(codes), np.concatenate([t, -t, [0.0]]))
    assert len(set(codes.tolist())) == 253
    # hand-picked codes: 1 = 0 0111 000, 448 = 0 1111 110, 2^-9 = 0 0000 001, -1.75 = 1 0111 110
    assert Q.e4m3_byte([1.0, 448.0, 2.0 ** -9, -1.75]).tolist() == [0x38, 0x7E, 0x01, 0xBE]


def test_e4m3_rounding_midpoints_and_saturation():
    t = _e4m3_table()
    mids = (t[:-1] + t[1:]) / 2
    r = Q.round_e4m3(mids)
    lo, hi = t[:-1], t[1:]
    # ties to the neighbour whose code is even
    even_lo = (Q.e4m3_byte(lo) & 1) == 0
    assert np.array_equal(r, np.where(even_lo, lo, hi))
    assert Q.round_e4m3([2.0 ** -10, 2.0 ** -11]).tolist() == [0.0, 0.0]      # half of 2^-9 ties to 0
    assert Q.round_e4m3([1000.0, 464.0, -1e9]).tolist() == [448.0, 448.0, -448.0]
    x = np.random.default_rng(0).uniform(-448, 448, 10000)
    r = Q.round_e4m3(x)
    # nearest: no table value is closer
    full = np.concatenate([-t[::-1], [0.0], t])
    best = full[np.abs(x[:, None] - full[None, :]).argmin(axis=1)]
    assert np.all(np.abs(x - r) <= np.abs(x - best))


def test_e4m3_blocks_scale_and_error():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((2, 200, 32)) * rng.uniform(0.01, 30, size=(2, 200, 1))).astype(np.float32)
    codes, scales = Q.quantize_blocks(x, 64, "e4m3")
    assert codes.dtype == np.uint8
    deq = Q.dequantize(codes, scales, 64, "e4m3")
    per_row = np.repeat(scales.astype(np.float64), 64, axis=-1)[..., :200, None]
    # relative 2^-4 for normals, half the subnormal step below 2^-6 (in code units)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, per_row * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(deq - x) <= bound)
    for b in range(4):   # the block's absmax element maps to 448
        assert np.all(np.abs(deq[..., b * 64:(b + 1) * 64, :]).max(axis=(-2, -1)) / scales[..., b] ==
                      pytest.approx(448.0, rel=1e-6))


def test_e4m3_attention_is_close_to_exact():
    rng = np.random.default_rng(2)
    n = 200
    q, k, v = (rng.standard_normal((1, 1, n, 128)).astype(np.float32) for _ in range(3))
    kept = np.ones((1, 1, 2, 4), dtype=bool)
    r8 = Q.block_sparse_attention_qk8_heads(q, k, v, kept, 128, 64, fmt="e4m3")
    r = A.block_sparse_attention_heads(q, k, v, kept, 128, 64)
    d = np.abs(r8["out"] - r["out"])
    assert d.max() < 5e-2 and d.mean() < 5e-3
