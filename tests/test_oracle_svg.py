"""Pins of the spatial / temporal head choice oracle (oracle.svg) against the
error-and-layout page's sections 3.3-5 and plain mathematics (CPU only)."""

import json
import os

import numpy as np
import pytest

from oracle import attention as A
from oracle import svg as S
from long_context_mean_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold():
    with open(os.path.join(GOLD, "worked_example.json")) as f:
        return json.load(f)


def test_pair_counts_on_the_worked_grid():
    g = _gold()
    T, H, W = g["grid"]
    assert int(S.element_mask(T, H, W, 0, S.SPATIAL).sum()) == g["pairs"]["spatial"]
    assert int(S.element_mask(T, H, W, 0, S.TEMPORAL).sum()) == g["pairs"]["temporal"]


@pytest.mark.parametrize("T,H,W,txt", [(3, 2, 5, 0), (5, 3, 2, 4), (2, 1, 1, 3)])
def test_pair_counts_closed_form(T, H, W, txt):
    """T P^2 and P T^2 video pairs (section 3.3) plus every pair that touches
    a text token: N^2 - nv^2 of them."""
    P, nv = H * W, T * H * W
    n = nv + txt
    assert int(S.element_mask(T, H, W, txt, S.SPATIAL).sum()) == T * P * P + n * n - nv * nv
    assert int(S.element_mask(T, H, W, txt, S.TEMPORAL).sum()) == P * T * T + n * n - nv * nv


def test_temporal_tile_ledger_before_and_after_reorder():
    """Section 4: 4x4 tiles on the 4x4x4 grid, 64 active tiles frame-major,
    16 after the token-major regrouping, utilisation 0.25 -> 1."""
    g = _gold()
    T, H, W = g["grid"]
    before = S.block_cover(S.element_mask(T, H, W, 0, S.TEMPORAL), 4, 4)
    after = S.head_block_mask(T, H, W, 0, S.TEMPORAL, 4, 4)
    assert int(before.sum()) == g["temporal_blocks_before"]["active_tiles"]
    assert int(after.sum()) == g["temporal_blocks_after"]["active_tiles"]
    assert int(before.sum()) * 16 == g["temporal_blocks_before"]["computed_pairs"]
    assert int(after.sum()) * 16 == g["temporal_blocks_after"]["computed_pairs"]


def test_token_major_perm_groups_positions_and_keeps_text():
    T, H, W, txt = 3, 2, 2, 2
    perm = S.token_major_perm(T, H, W, txt)
    P = H * W
    assert sorted(perm.tolist()) == list(range(T * P + txt))
    for n in range(T * P):
        p, t = divmod(n, T)
        assert perm[n] == t * P + p
    assert perm[T * P:].tolist() == [T * P, T * P + 1]


def _interval_rule(nv, n, group, bq, bk):
    """Closed form of the block cover: a tile is kept iff it reaches a text
    token or the group ranges of its rows and columns intersect."""
    nqb, nkb = -(-n // bq), -(-n // bk)
    out = np.zeros((nqb, nkb), dtype=bool)
    for qb in range(nqb):
        i0, i1 = qb * bq, min(n, (qb + 1) * bq) - 1
        for kb in range(nkb):
            j0, j1 = kb * bk, min(n, (kb + 1) * bk) - 1
            out[qb, kb] = i1 >= nv or j1 >= nv or (i0 // group <= j1 // group and j0 // group <= i1 // group)
    return out


@pytest.mark.parametrize("seed", range(6))
def test_block_cover_matches_interval_rule(seed):
    rng = np.random.default_rng(seed)
    T, H, W = (int(x) for x in rng.integers(1, 6, size=3))
    txt = int(rng.integers(0, 7))
    bq, bk = (int(x) for x in rng.integers(1, 9, size=2))
    nv = T * H * W
    n = nv + txt
    for kind, group in ((S.SPATIAL, H * W), (S.TEMPORAL, T)):
        got = S.head_block_mask(T, H, W, txt, kind, bq, bk)
        assert np.array_equal(got, _interval_rule(nv, n, group, bq, bk)), (kind, T, H, W, txt, bq, bk)


def test_aligned_candidates_equal_element_masked_softmax():
    """With tiles of one frame (spatial) or one position (temporal), the
    block-sparse candidate is the restricted softmax of section 3.1 on the
    element mask, in the original order (the temporal one through the
    permutation of section 3.4)."""
    ex = inputs.worked_example_inputs()
    T, P = ex["T"], ex["P"]
    q, k, v = ex["q"], ex["k"], ex["v"]
    for h in range(2):
        for kind, blk in ((S.SPATIAL, P), (S.TEMPORAL, T)):
            out, lse = S.candidate_attention(q[h], k[h], v, 4, 4, 4, 0, kind, blk, blk)
            y, _, ref_lse = A.masked_attention(q[h], k[h], v, S.element_mask(4, 4, 4, 0, kind))
            assert np.max(np.abs(out - y)) < 1e-13
            assert np.max(np.abs(lse - ref_lse)) < 1e-12


def test_text_rows_see_everything():
    """A text query's candidate output is dense attention's (every key kept)."""
    rng = np.random.default_rng(3)
    T, H, W, txt = 2, 2, 3, 5
    n = T * H * W + txt
    q, k, v = rng.normal(size=(3, n, 8))
    dense = A.dense_attention(q, k, v)[0]
    for kind in (S.SPATIAL, S.TEMPORAL):
        out, _ = S.candidate_attention(q, k, v, T, H, W, txt, kind, 4, 4)
        assert np.max(np.abs(out[T * H * W:] - dense[T * H * W:])) < 1e-13


def test_worked_example_selects_spatial_then_temporal():
    """Section 5: on the two synthetic heads the argmin picks the spatial
    candidate for head 0 and the temporal one for head 1; the page's sampled
    MSEs differ by more than four orders of magnitude between candidates."""
    ex = inputs.worked_example_inputs()
    q, k = ex["q"], ex["k"]
    v = np.stack([ex["v"], ex["v"]])
    rows = np.arange(64)
    choice, mse = S.select_heads(q, k, v, 4, 4, 4, 0, 4, 4, rows)
    assert choice.tolist() == [S.SPATIAL, S.TEMPORAL]
    assert mse[S.TEMPORAL, 0] > 1e4 * mse[S.SPATIAL, 0]
    assert mse[S.SPATIAL, 1] > 1e4 * mse[S.TEMPORAL, 1]
    # All 64 rows: the MSE is the plain mean over every output (section 4).
    dense0 = A.dense_attention(q[0], k[0], ex["v"])[0]
    out0, _ = S.candidate_attention(q[0], k[0], ex["v"], 4, 4, 4, 0, S.SPATIAL, 4, 4)
    assert mse[S.SPATIAL, 0] == pytest.approx(float(np.mean((dense0 - out0) ** 2)), rel=1e-12)


def test_sampled_mse_counts_repeats():
    ref = np.array([[0.0, 0.0], [1.0, 1.0], [2.0, 2.0]])
    x = np.zeros_like(ref)
    assert S.sampled_mse(ref, x, [1, 1, 2]) == pytest.approx((1 + 1 + 4) / 3)
    assert S.sampled_mse(ref, x, []) == 0.0


def test_svg_attention_follows_the_choice():
    ex = inputs.worked_example_inputs()
    q, k = ex["q"], ex["k"]
    v = np.stack([ex["v"], ex["v"]])
    out, lse = S.svg_attention(q, k, v, [S.TEMPORAL, S.SPATIAL], 4, 4, 4, 0, 4, 4)
    o0, l0 = S.candidate_attention(q[0], k[0], v[0], 4, 4, 4, 0, S.TEMPORAL, 4, 4)
    o1, l1 = S.candidate_attention(q[1], k[1], v[1], 4, 4, 4, 0, S.SPATIAL, 4, 4)
    assert np.array_equal(out[0], o0) and np.array_equal(out[1], o1)
    assert np.array_equal(lse[0], l0) and np.array_equal(lse[1], l1)
