"""fp64-free (integer) token layouts: identity, [t,h,w] windows, Hilbert curve.

TEST INFRASTRUCTURE ONLY (see the package header).

Token numbering before any reorder is raster frame-major over the video
latent, i = t*H*W + h*W + w ([P1] section 3.3), with ``txt_len`` text tokens
appended after the video tokens.  A permutation ``perm`` maps an output
position n to the source index it takes (y[n] = x[perm[n]]); ``inv`` is its
inverse (x[i] = y[inv[i]]), the "inverse reorder" of [P1] section 3.4 and
[P3] section 2.5.

Readings (the pages are silent on these):
* The first ``sink_frames`` frames (the first-frame sink of [P2]) stay at the
  front in raster order and are not reordered; text tokens stay last and are
  not reordered ([P3] section 2.5 permutes visual tokens only; [P1] section 5
  keeps trailing context tokens in place).
* Window mode ([P2] "[t, h, w] 三维窗口重排"): windows of size [wt, wh, ww]
  tile the remaining frames; edge windows are smaller (no padding).  Windows
  are visited in raster order of their (t, h, w) window coordinates and the
  tokens inside a window in raster order.
* Hilbert mode ([P3] section 2.5): the curve is the one of J. Skilling,
  "Programming the Hilbert curve", AIP Conf. Proc. 707 (2004) -- the
  axes-to-transpose algorithm on the 2^b cube with b = ceil(log2(max dim)),
  axis order (t, h, w) with t most significant; the present points are
  sorted by their curve index.

Parity: window and identity are pinned by closed forms ([P1] section 4:
window [T,1,1] equals the stable argsort by pixel; a window covering the
whole grid is the identity; the 4x4 temporal ledger goes from 64 to 16
tiles).  The Hilbert index is pinned, in two dimensions, to an independent
construction: the classic rotate-and-reflect Hilbert curve, equal index for
index on every grid up to 64 x 64 (Skilling's algorithm is generic in the
number of axes, so the same inversion, exchange, Gray-encode and interleave
steps serve both).  In three dimensions it is pinned by the defining
properties of a Hilbert curve: bijection and unit steps on full cubes, start
at the origin and end at (2^b - 1, 0, 0), octants in binary-reflected Gray
order with t most significant, and exact self-similarity (every order is
eight isometric copies of the order below, by the same eight isometries).
The pages name no Hilbert variant; among the three-axis variants this one is
Skilling's by the algorithm the two-dimensional pin checks.
"""

from __future__ import annotations

import numpy as np


def _finish(perm: np.ndarray):
    perm = np.asarray(perm, dtype=np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int64)
    return perm, inv


def identity_perm(n: int):
    return _finish(np.arange(n))


def window_perm(T: int, H: int, W: int, win, sink_frames: int = 0, txt_len: int = 0):
    """[t,h,w] window reorder of the frames after the sink ([P2])."""
    wt, wh, ww = (int(x) for x in win)
    if min(wt, wh, ww) <= 0:
        raise ValueError("window sizes must be positive")
    P = H * W
    head = list(range(sink_frames * P))
    body = []
    for t0 in range(sink_frames, T, wt):
        for h0 in range(0, H, wh):
            for w0 in range(0, W, ww):
                for t in range(t0, min(T, t0 + wt)):
                    for h in range(h0, min(H, h0 + wh)):
                        for w in range(w0, min(W, w0 + ww)):
                            body.append(t * P + h * W + w)
    tail = list(range(T * P, T * P + txt_len))
    return _finish(head + body + tail)


def hilbert_bits(*dims) -> int:
    m = max(int(x) for x in dims)
    b = 1
    while (1 << b) < m:
        b += 1
    return b


def hilbert_index(coords, bits: int) -> np.ndarray:
    """Hilbert index of integer points on the 2^bits cube (Skilling 2004).

    coords: int array [npts, ndim], axis 0 of the point is the most
    significant.  Steps: (1) undo the excess work -- for each bit Q from the
    top down to 2, for each axis i, either invert the low bits of axis 0 (if
    bit Q of axis i is set) or exchange the low bits of axes 0 and i;
    (2) Gray-encode across the axes; (3) interleave the bits of the
    transposed form, most significant bit plane first, axis 0 first.
    """
    x = np.array(coords, dtype=np.int64, copy=True)
    npts, n = x.shape
    top = 1 << (bits - 1)
    q = top
    while q > 1:
        p = q - 1
        for i in range(n):
            has = (x[:, i] & q) != 0
            x[has, 0] ^= p
            t = (x[~has, 0] ^ x[~has, i]) & p
            x[~has, 0] ^= t
            x[~has, i] ^= t
        q >>= 1
    for i in range(1, n):
        x[:, i] ^= x[:, i - 1]
    t = np.zeros(npts, dtype=np.int64)
    q = top
    while q > 1:
        t = np.where((x[:, n - 1] & q) != 0, t ^ (q - 1), t)
        q >>= 1
    for i in range(n):
        x[:, i] ^= t
    index = np.zeros(npts, dtype=np.int64)
    for b in range(bits - 1, -1, -1):
        for i in range(n):
            index = (index << 1) | ((x[:, i] >> b) & 1)
    return index


def hilbert_perm(T: int, H: int, W: int, sink_frames: int = 0, txt_len: int = 0):
    """Hilbert-curve reorder of the frames after the sink ([P3] section 2.5)."""
    P = H * W
    Tr = T - sink_frames
    head = np.arange(sink_frames * P)
    if Tr > 0:
        t, h, w = np.meshgrid(np.arange(Tr), np.arange(H), np.arange(W), indexing="ij")
        pts = np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1)
        key = hilbert_index(pts, hilbert_bits(Tr, H, W))
        src = (pts[:, 0] + sink_frames) * P + pts[:, 1] * W + pts[:, 2]
        body = src[np.argsort(key, kind="stable")]
    else:
        body = np.zeros(0, dtype=np.int64)
    tail = np.arange(T * P, T * P + txt_len)
    return _finish(np.concatenate([head, body, tail]))


def build_layout(mode: str, T: int, H: int, W: int, win=(1, 1, 1), sink_frames=0, txt_len=0):
    n = T * H * W + txt_len
    if mode == "identity":
        return identity_perm(n)
    if mode == "window":
        return window_perm(T, H, W, win, sink_frames, txt_len)
    if mode == "hilbert":
        return hilbert_perm(T, H, W, sink_frames, txt_len)
    raise ValueError(mode)


def reorder(x: np.ndarray, perm: np.ndarray, axis: int = -2) -> np.ndarray:
    """y[..., n, :] = x[..., perm[n], :] (Q, K, V reorder)."""
    return np.take(x, perm, axis=axis)


def unreorder(y: np.ndarray, perm: np.ndarray, axis: int = -2) -> np.ndarray:
    """x[..., perm[n], :] = y[..., n, :] (inverse reorder of O and LSE)."""
    x = np.empty_like(y)
    idx = [slice(None)] * y.ndim
    idx[axis] = perm
    x[tuple(idx)] = y
    return x
