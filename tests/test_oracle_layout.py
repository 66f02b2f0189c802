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


def _classic_hilbert_d(n, x, y):
    """Distance along the classic two-dimensional Hilbert curve on an n x n
    grid (n a power of two): at each scale s the quadrant (rx, ry) gives
    s*s*((3*rx) ^ ry), then the point is reflected and its axes swapped
    into the quadrant's frame.  Written independently of Skilling's
    transpose algorithm; the two must agree in two dimensions, where the
    Hilbert curve from (0, 0) to (n-1, 0) is unique."""
    d = 0
    s = n // 2
    while s > 0:
        rx = 1 if x & s else 0
        ry = 1 if y & s else 0
        d += s * s * ((3 * rx) ^ ry)
        if ry == 0:
            if rx == 1:
                x, y = n - 1 - x, n - 1 - y
            x, y = y, x
        s //= 2
    return d


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6])
def test_hilbert_2d_equals_the_classic_construction(bits):
    """Skilling's algorithm is generic in the number of axes: in two
    dimensions it must give exactly the classic Hilbert curve (the same
    loops -- the inversion/exchange pass, the Gray encoding, the bit
    interleave -- that serve the three-axis layout)."""
    n = 1 << bits
    x, y = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    pts = np.stack([x.ravel(), y.ravel()], axis=1)
    idx = Y.hilbert_index(pts, bits)
    ref = np.array([_classic_hilbert_d(n, int(a), int(b)) for a, b in pts])
    assert np.array_equal(idx, ref)


def _curve3(bits):
    n = 1 << bits
    t, h, w = np.meshgrid(np.arange(n), np.arange(n), np.arange(n), indexing="ij")
    pts = np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1)
    return pts[np.argsort(Y.hilbert_index(pts, bits))]


def _octant_isometries(bits):
    """For each of the 8 octants of the order-`bits` curve (in curve order):
    the cube isometry (axis permutation, reflections) that maps the
    order-(bits-1) curve onto the octant's piece of the curve."""
    import itertools
    big, small = _curve3(bits), _curve3(bits - 1)
    m = (1 << (bits - 1)) - 1
    L = len(small)
    found = []
    for c in range(8):
        piece = big[c * L:(c + 1) * L]
        rel = piece - (piece[0] // (m + 1)) * (m + 1)
        match = []
        for perm in itertools.permutations(range(3)):
            for flips in itertools.product([0, 1], repeat=3):
                q = small[:, list(perm)].copy()
                for a in range(3):
                    if flips[a]:
                        q[:, a] = m - q[:, a]
                if np.array_equal(q, rel):
                    match.append((perm, flips))
        assert len(match) == 1            # each piece is one isometric copy
        found.append(match[0])
    return found


def test_hilbert_3d_gray_order_end_corner_and_self_similarity():
    """Three axes: at every order the curve runs from the origin to
    (2^b - 1, 0, 0), visits the octants in binary-reflected Gray-code order
    of their (t, h, w) bits with t most significant, and each octant holds an
    isometric copy of the curve one order down, by the same eight isometries
    at every order (one generator, as a Hilbert curve is defined)."""
    gray = [(g >> 2 & 1, g >> 1 & 1, g & 1) for g in (i ^ (i >> 1) for i in range(8))]
    gen = None
    for bits in range(1, 6):
        path = _curve3(bits)
        n = 1 << bits
        assert tuple(path[0]) == (0, 0, 0) and tuple(path[-1]) == (n - 1, 0, 0)
        octs = [tuple(int(v) for v in p) for p in path[::len(path) // 8] // max(1, n // 2)]
        assert octs == gray
        if bits >= 2:
            iso = _octant_isometries(bits)
            gen = iso if gen is None else gen
            assert iso == gen
