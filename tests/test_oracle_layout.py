"""Pins of the layout oracle (CPU only)."""

import numpy as np
import pytest

from oracle import layout as Y
from oracle import ledger as L


def test_window_t_only_equals_stable_argsort_by_pixel():
    """Window [T,1,1] groups each position's frames together: the stable
    argsort by pixel index of the worked example ([P1] section 4)."""
    T, H, W = 4, 4, 4
    perm, inv = Y.window_perm(T, H, W, (T, 1, 1))
    pixel = np.tile(np.arange(H * W), T)
    assert np.array_equal(perm, np.argsort(pixel, kind="stable"))
    assert np.array_equal(perm[inv], np.arange(T * H * W))


def test_window_reorder_block_ledger_64_to_16():
    g = {"before": (64, 1024, 0.25), "after": (16, 256, 1.0)}
    m = L.video_masks(4, 4, 4)["temporal"]
    perm, _ = Y.window_perm(4, 4, 4, (4, 1, 1))
    before = L.block_cost(m, 4)
    after = L.block_cost(m[np.ix_(perm, perm)], 4)
    assert (before["active_tiles"], before["computed_pairs"], before["utilization"]) == g["before"]
    assert (after["active_tiles"], after["computed_pairs"], after["utilization"]) == g["after"]


def test_window_whole_grid_is_identity_and_text_sink_fixed():
    perm, _ = Y.window_perm(3, 5, 7, (3, 5, 7))
    assert np.array_equal(perm, np.arange(105))
    perm, _ = Y.window_perm(5, 4, 6, (2, 3, 4), sink_frames=1, txt_len=9)
    P = 24
    assert np.array_equal(perm[:P], np.arange(P))
    assert np.array_equal(perm[-9:], np.arange(5 * P, 5 * P + 9))
    assert sorted(perm) == list(range(5 * P + 9))


def test_window_edge_windows_are_smaller():
    """H=5 with wh=2 leaves a one-row edge window; tokens inside a window
    are raster ordered, windows raster ordered."""
    perm, _ = Y.window_perm(1, 5, 3, (1, 2, 3))
    expect = [0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14]
    assert list(perm) == expect  # ww = W: rows stay contiguous
    perm, _ = Y.window_perm(1, 3, 5, (1, 2, 2))
    # windows: (h0=0,w0=0) -> (0,0),(0,1),(1,0),(1,1) = 0,1,5,6 ; (0,2)->2,3,7,8 ;
    # (0,4)->4,9 ; (2,0)->10,11 ; (2,2)->12,13 ; (2,4)->14
    assert list(perm) == [0, 1, 5, 6, 2, 3, 7, 8, 4, 9, 10, 11, 12, 13, 14]


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_hilbert_full_cube_unit_steps(bits):
    n = 1 << bits
    t, h, w = np.meshgrid(np.arange(n), np.arange(n), np.arange(n), indexing="ij")
    pts = np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1)
    idx = Y.hilbert_index(pts, bits)
    assert np.array_equal(np.sort(idx), np.arange(n ** 3))        # bijection
    path = pts[np.argsort(idx)]
    steps = np.abs(np.diff(path, axis=0)).sum(axis=1)
    assert np.all(steps == 1)                                      # continuity
    assert np.array_equal(path[0], [0, 0, 0])                      # starts at origin


def test_hilbert_2d_unit_steps_and_quadrants():
    n = 16
    x, y = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    pts = np.stack([x.ravel(), y.ravel()], axis=1)
    idx = Y.hilbert_index(pts, 4)
    path = pts[np.argsort(idx)]
    assert np.all(np.abs(np.diff(path, axis=0)).sum(axis=1) == 1)
    # Each aligned quarter of the curve fills one 8x8 quadrant.
    for qd in range(4):
        seg = path[qd * 64:(qd + 1) * 64] // 8
        assert len({tuple(p) for p in seg}) == 1


def test_hilbert_perm_non_cubic_box_is_bijection_with_locality():
    T, H, W = 6, 5, 7
    perm, inv = Y.hilbert_perm(T, H, W, sink_frames=1, txt_len=3)
    n = T * H * W + 3
    assert sorted(perm) == list(range(n))
    assert np.array_equal(perm[:35], np.arange(35))
    assert np.array_equal(perm[-3:], np.arange(n - 3, n))
    # Locality: the average coordinate jump along the curve is far below raster's.
    body = perm[35:-3] - 35
    coords = np.stack(np.unravel_index(body, (T - 1, H, W)), axis=1)
    jump = np.abs(np.diff(coords, axis=0)).sum(axis=1).mean()
    raster = np.stack(np.unravel_index(np.arange(len(body)), (T - 1, H, W)), axis=1)
    raster_jump = np.abs(np.diff(raster, axis=0)).sum(axis=1).mean()
    assert jump < 0.8 * raster_jump


def test_reorder_unreorder_round_trip():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(2, 3, 50, 4))
    perm, inv = Y.build_layout("window", 2, 5, 5, (2, 2, 2), 0, 0)
    y = Y.reorder(x, perm)
    assert np.array_equal(Y.unreorder(y, perm), x)
    assert np.array_equal(np.take(y, inv, axis=-2), x)
