"""Pins of the ledgers: pair counts and densities of the toy video grid."""

import numpy as np
import pytest

from oracle import ledger as L


@pytest.mark.parametrize("T,H,W", [(4, 4, 4), (3, 2, 5), (6, 3, 3)])
def test_pair_counts_and_densities(T, H, W):
    P = H * W
    m = L.video_masks(T, H, W)
    assert int(m["full"].sum()) == T * T * P * P
    assert int(m["spatial"].sum()) == T * P * P
    assert int(m["temporal"].sum()) == P * T * T
    assert m["spatial"].mean() == pytest.approx(1 / T, abs=1e-15)
    assert m["temporal"].mean() == pytest.approx(1 / P, abs=1e-15)
    assert m["union"].mean() == pytest.approx((P + T - 1) / (T * P), abs=1e-15)


def test_union_density_toy_is_19_over_64():
    assert L.video_masks(4, 4, 4)["union"].mean() == 19 / 64


def test_block_cost_counts():
    m = np.zeros((8, 8), dtype=bool)
    m[0, 0] = m[5, 6] = True
    c = L.block_cost(m, 4)
    assert c == {"useful_pairs": 2, "active_tiles": 2, "computed_pairs": 32, "utilization": 2 / 32}


def test_coverage_summary_window_vs_global():
    g = L.coverage_summary(np.tril(np.ones((8, 8), dtype=bool)), 3)
    w = L.coverage_summary(L.selective_mask(8, 3, []), 3)
    assert g["score_count"] == 36 and g["density"] == 1.0 and g["long_range_coverage"] == 1.0
    assert w["long_range_coverage"] == 0.0 and 0 < w["density"] < 1
    s = L.coverage_summary(L.selective_mask(8, 2, [0]), 3)
    assert s["long_range_coverage"] > 0
