"""Pins of the mask-prediction oracle (CPU only)."""

import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

from oracle import ledger as L
from oracle import predict as Pr

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# Pooling and the similarity guard
# --------------------------------------------------------------------------

def test_pool_uses_true_count_of_tail_block():
    x = np.arange(10.0)[:, None] * np.array([[1.0, -2.0]])
    m = Pr.pool_blocks(x, 4)
    assert m.shape == (3, 2)
    assert np.allclose(m[2], [8.5, -17.0])        # mean of rows 8, 9 only


def test_cossim_closed_form_and_special_cases():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(13, 7))
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    closed = np.linalg.norm(u.sum(axis=0)) ** 2 / 13 ** 2
    assert Pr.cossim_block(x) == pytest.approx(closed, abs=1e-14)
    same = np.tile(rng.normal(size=(1, 5)) * 3.0, (6, 1))
    assert Pr.cossim_block(same) == pytest.approx(1.0, abs=1e-14)
    ortho = np.linalg.qr(rng.normal(size=(8, 8)))[0] * 4.0
    assert Pr.cossim_block(ortho) == pytest.approx(1.0 / 8, abs=1e-14)
    # Scale invariance per token, and a zero vector contributes 0.
    assert Pr.cossim_block(x * rng.uniform(0.1, 9, size=(13, 1))) == pytest.approx(closed, abs=1e-13)
    z = np.vstack([same, np.zeros((2, 5))])
    assert Pr.cossim_block(z) == pytest.approx(36 / 64, abs=1e-14)


# --------------------------------------------------------------------------
# TopCdf
# --------------------------------------------------------------------------

def test_topcdf_teaching_example():
    """[0.6, 0.3, 0.1] with tau = 0.8 keeps the first two (the reading that
    keeps the element which crosses tau)."""
    kept, c = Pr.topcdf(np.array([0.3, 0.6, 0.1]), 0.8)
    assert kept.tolist() == [True, True, False]
    assert np.allclose(c, [0.6, 0.0, 0.9])


def test_topcdf_limits():
    rng = np.random.default_rng(1)
    p = softmax(rng.normal(size=40))
    kept, _ = Pr.topcdf(p, 1e-9)
    assert kept.sum() == 1 and kept[np.argmax(p)]
    p2 = p.copy()
    p2[[3, 9]] = 0.0
    kept, _ = Pr.topcdf(p2, 1.0)
    assert np.array_equal(kept, p2 > 0)


def test_topcdf_ties_lower_index_first():
    kept, _ = Pr.topcdf(np.array([0.25, 0.25, 0.25, 0.25]), 0.5)
    assert kept.tolist() == [True, True, False, False]


def test_topcdf_is_smallest_prefix_reaching_tau_brute_force():
    """Exhaustive search: the kept set is the smallest set, among sets made
    of the largest entries, whose mass reaches tau."""
    rng = np.random.default_rng(2)
    for _ in range(200):
        n = rng.integers(1, 8)
        p = rng.random(n) ** 3
        p /= p.sum()
        tau = rng.uniform(0.05, 1.0)
        kept, _ = Pr.topcdf(p, tau)
        best = None
        for r in range(1, n + 1):
            for combo in itertools.combinations(range(n), r):
                if p[list(combo)].sum() >= tau * p.sum() - 1e-15:
                    best = r
                    break
            if best is not None:
                break
        assert kept.sum() == best
        # the kept ones are the largest ones
        assert p[kept].min() >= p[~kept].max(initial=-1.0)


def test_compressed_probs_is_library_softmax_over_eligible():
    rng = np.random.default_rng(3)
    qh, kh = rng.normal(size=8), rng.normal(size=(11, 8))
    elig = rng.random(11) < 0.6
    elig[0] = True
    p = Pr.compressed_probs(qh, kh, elig, 8)
    assert np.allclose(p[elig], softmax(kh[elig] @ qh / math.sqrt(8)), atol=1e-15)
    assert np.all(p[~elig] == 0)


# --------------------------------------------------------------------------
# Windows, anchors and causal validity: the pages' unit tests
# --------------------------------------------------------------------------

def test_local_and_block_masks_reproduce_printed_unit_tests():
    g = _gold("access_patterns.json")
    m = L.local_causal_mask(5, 2)
    assert all(m[i, j] for i, j in g["local_window_5_2"]["visible"])
    assert not any(m[i, j] for i, j in g["local_window_5_2"]["hidden"])
    bm = L.block_pair_mask(4, 2, [tuple(p) for p in g["block_pairs_4_2"]["pairs"]])
    assert all(bm[i, j] for i, j in g["block_pairs_4_2"]["visible"])
    assert not any(bm[i, j] for i, j in g["block_pairs_4_2"]["hidden"])
    assert not L.block_pair_mask(4, 2, []).any()
    with pytest.raises(ValueError):
        L.block_pair_mask(4, 2, [(2, 0)])
    with pytest.raises(ValueError):
        L.block_pair_mask(4, 2, [(0, 1)])
    assert L.block_pair_mask(4, 2, [(0, 1)], causal=False)[0, 2]
    assert L.access_summary(L.local_causal_mask(4, 2)) == g["summary_local_4_2"]
    sel = L.selective_mask(8, g["selective_8"]["window"], g["selective_8"]["anchors"])
    assert all(sel[i, j] for i, j in g["selective_8"]["visible"])
    win = L.selective_mask(8, 3, [])
    assert all(win[i, j] for i, j in g["window_8_3"]["visible"])
    assert not any(win[i, j] for i, j in g["window_8_3"]["hidden"])


def test_sliding_window_pair_count_and_reduction():
    g = _gold("access_patterns.json")
    for L_, w in [(8, 3), (20, 5), (33, 1)]:
        assert int(L.local_causal_mask(L_, w).sum()) == L.sliding_window_pairs(L_, w)
    red = 100 * (1 - L.sliding_window_pairs(2048, 256) / (2048 * 2049 / 2))
    assert round(red, 2) == g["sliding_reduction_L2048_w256_percent"]


def _brute_block_window(n, bq, bk, w):
    nqb, nkb = -(-n // bq), -(-n // bk)
    out = np.zeros((nqb, nkb), dtype=bool)
    for i in range(n):
        for j in range(n):
            if 0 <= i - j < w:
                out[i // bq, j // bk] = True
    return out


@pytest.mark.parametrize("n,bq,bk,w", [(100, 16, 8, 20), (77, 32, 16, 5), (64, 16, 16, 1), (90, 8, 32, 40)])
def test_block_window_and_causal_validity_brute_force(n, bq, bk, w):
    rng = np.random.default_rng(n)
    q = rng.normal(size=(1, n, 4))
    r = Pr.predict_mask_batch(q, q, bq, bk, tau=1e-9, theta=0.0, causal=True, local_window=w)
    assert np.array_equal(r["mask"][0] | r["top"][0], r["mask"][0])
    brute_w = _brute_block_window(n, bq, bk, w)
    # everything the window opens is kept; kept = window | top-1
    assert np.array_equal(r["mask"][0] & ~r["top"][0], brute_w & ~r["top"][0])
    valid = np.zeros_like(brute_w)
    for i in range(n):
        for j in range(i + 1):
            valid[i // bq, j // bk] = True
    assert np.array_equal(r["valid"], valid)


def test_forced_rows_cols_sink_text_anchors():
    rng = np.random.default_rng(4)
    n, d, bq, bk = 96, 8, 16, 8
    x = rng.normal(size=(2, n, d))
    # Make q-block 2 and k-block 5 highly coherent (high similarity), the rest
    # random (low similarity ~ 1/b), so theta = 0.5 forces all but those.
    x[:, 32:48] = rng.normal(size=(1, 1, d)) + 0.01 * rng.normal(size=(2, 16, d))
    x[:, 40:48] = x[:, 40:48]
    r = Pr.predict_mask_batch(x, x, bq, bk, tau=0.5, theta=0.5)
    assert not r["forced_rows"][0, 2] and r["forced_rows"][0, 0]
    assert np.all(r["mask"][0, r["forced_rows"][0]])
    assert np.all(r["mask"][0][:, r["forced_cols"][0]])
    r2 = Pr.predict_mask_batch(x, x, bq, bk, tau=1e-9, theta=0.0, sink_tokens=20,
                               txt_len=10, anchor_tokens=9)
    m = r2["mask"][0]
    assert m[0].all() and m[1].all()            # q rows 0..31 hold sink tokens
    assert m[:, 0].all() and m[:, 1].all() and m[:, 2].all()   # sink 0..19 -> k blocks 0..2
    assert m[-1].all()                          # last q-block holds text
    assert m[:, -2].all() and m[:, -1].all()    # text 86..95 -> k blocks 10, 11


def test_gqa_uses_group_kv_head():
    rng = np.random.default_rng(5)
    n, d = 64, 8
    q = rng.normal(size=(4, n, d))
    k = rng.normal(size=(2, n, d))
    r = Pr.predict_mask_batch(q, k, 16, 16, tau=0.3, theta=0.0)
    r1 = Pr.predict_mask_batch(q[2:4], k[1:2], 16, 16, tau=0.3, theta=0.0)
    assert np.array_equal(r["mask"][2:4], r1["mask"])


def test_csr_and_order():
    m = np.array([[[1, 0, 1], [0, 0, 1]], [[1, 1, 1], [0, 1, 0]]], dtype=bool)
    c = Pr.mask_to_csr(m)
    assert c["row_ptr"].tolist() == [0, 2, 3, 6, 7]
    assert c["col_idx"].tolist() == [0, 2, 2, 0, 1, 2, 1]
    assert c["order"].tolist() == [2, 0, 1, 3]
    assert c["kept_total"] == 7


def test_work_order_in_head_groups():
    # 2 heads x 2 query blocks, counts [1, 3 | 2, 2]: one global order puts
    # the 3-block row first; groups of one head sort each head's rows alone.
    m = np.array([[[1, 0, 0], [1, 1, 1]], [[1, 1, 0], [0, 1, 1]]], dtype=bool)
    assert Pr.mask_to_csr(m)["order"].tolist() == [1, 2, 3, 0]
    assert Pr.mask_to_csr(m, order_group=1)["order"].tolist() == [1, 0, 2, 3]
    assert Pr.mask_to_csr(m, order_group=2)["order"].tolist() == [1, 2, 3, 0]
    # a group larger than the heads is one global order; ragged last group
    m3 = np.concatenate([m, m[:1]], axis=0)            # 3 heads, counts [1,3 | 2,2 | 1,3]
    assert Pr.mask_to_csr(m3, order_group=2)["order"].tolist() == [1, 2, 3, 0, 5, 4]
    assert Pr.mask_to_csr(m3, order_group=8)["order"].tolist() == Pr.mask_to_csr(m3)["order"].tolist()


def test_empty_rows_element_level():
    # causal, bq = 4 > bk = 2: q-block 1 (rows 4..7) keeping only k-block 3
    # (keys 6, 7) leaves rows 4 and 5 with nothing.
    m = np.zeros((2, 4), dtype=bool)
    m[0, 0] = True
    m[1, 3] = True
    bad = Pr.empty_rows(m, 8, 4, 2, causal=True)
    assert bad.tolist() == [False, True]
    m[1, 2] = True
    assert Pr.empty_rows(m, 8, 4, 2, causal=True).tolist() == [False, False]
    assert Pr.empty_rows(np.zeros((2, 4), dtype=bool), 8, 4, 2, causal=False).tolist() == [True, True]
