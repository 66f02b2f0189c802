"""Integer ledgers of allowed query/key pairs, block occupancy and coverage.

TEST INFRASTRUCTURE ONLY (see the package header).

* ``video_masks`` -- the spatial (same frame), temporal (same position) and
  union masks of [P1] section 3.3 on a frame-major [T, H, W] grid.
* ``block_cost`` -- the block-occupancy ledger of [P1] section 4: a block is
  computed whole as soon as it holds one allowed pair.
* ``local_causal_mask``, ``block_pair_mask``, ``access_summary`` -- [P4]
  Step 4 (window visibility, block pairs with causal filter, pair ledger).
* ``selective_mask``, ``coverage_summary`` -- [P5] Steps 2 and 4 (window
  plus anchors; visible keys, long-range coverage, density against the
  causal global mask).

Pins: the 4096 / 1024 / 256 pair counts and the densities 1/T, 1/P,
(P+T-1)/(TP) of [P1] section 3.3; the 64 -> 16 tile ledger of [P1]
section 4; the unit tests printed on [P4] and [P5]; the sliding-window pair
count wL - w(w-1)/2 of [P4] Step 2 and its 76.57% reduction at L = 2048,
w = 256 ([P4] section 5.4).
"""

from __future__ import annotations

import numpy as np


def video_masks(T: int, H: int, W: int):
    P = H * W
    n = T * P
    frame = np.repeat(np.arange(T), P)
    pixel = np.tile(np.arange(P), T)
    spatial = frame[:, None] == frame[None, :]
    temporal = pixel[:, None] == pixel[None, :]
    return {"full": np.ones((n, n), dtype=bool), "spatial": spatial,
            "temporal": temporal, "union": spatial | temporal,
            "frame": frame, "pixel": pixel}


def block_cost(mask, block):
    """Active tiles, computed pairs and utilization of a square token mask
    cut into block x block tiles."""
    mask = np.asarray(mask, dtype=bool)
    n = mask.shape[0]
    if n % block:
        raise ValueError("mask size must be a multiple of the block")
    nb = n // block
    active = 0
    for bi in range(nb):
        for bj in range(nb):
            if mask[bi * block:(bi + 1) * block, bj * block:(bj + 1) * block].any():
                active += 1
    pairs = int(mask.sum())
    computed = active * block * block
    return {"useful_pairs": pairs, "active_tiles": active,
            "computed_pairs": computed, "utilization": pairs / computed}


def local_causal_mask(seq_len: int, window: int):
    """key <= query and query - key < window ([P4] Step 4)."""
    if seq_len <= 0 or window <= 0:
        raise ValueError("seq_len and window must be positive")
    mask = np.zeros((seq_len, seq_len), dtype=bool)
    for i in range(seq_len):
        for j in range(seq_len):
            mask[i, j] = (j <= i) and (i - j < window)
    return mask


def block_pair_mask(seq_len: int, block: int, pairs, causal=True):
    """Token mask opening the listed (query block, key block) pairs, with the
    causal filter applied element-wise; out-of-range or (when causal)
    future block pairs are rejected ([P4] Step 4)."""
    if seq_len <= 0 or block <= 0:
        raise ValueError("seq_len and block must be positive")
    nb = -(-seq_len // block)
    mask = np.zeros((seq_len, seq_len), dtype=bool)
    for qb, kb in pairs:
        if not (0 <= qb < nb and 0 <= kb < nb):
            raise ValueError("block pair out of range")
        if causal and kb > qb:
            raise ValueError("causal block mask cannot open a future block")
        mask[qb * block:min(seq_len, (qb + 1) * block),
             kb * block:min(seq_len, (kb + 1) * block)] = True
    if causal:
        mask &= np.tril(np.ones((seq_len, seq_len), dtype=bool))
    return mask


def access_summary(mask):
    mask = np.asarray(mask, dtype=bool)
    vis = int(mask.sum())
    return {"visible_pairs": vis, "total_pairs": int(mask.size), "density": vis / mask.size}


def sliding_window_pairs(L: int, w: int) -> int:
    """Closed form wL - w(w-1)/2 for L >= w ([P4] Step 2)."""
    return w * L - w * (w - 1) // 2


def selective_mask(seq_len: int, window: int, anchors):
    """Causal window of ``window`` most recent keys plus anchor keys ([P5])."""
    anchors = set(int(a) for a in anchors)
    mask = np.zeros((seq_len, seq_len), dtype=bool)
    for i in range(seq_len):
        for j in range(i + 1):
            mask[i, j] = (j >= i - window + 1) or (j in anchors)
    return mask


def coverage_summary(mask, local_window: int):
    """visible_keys_mean, score_count, long_range_coverage (allowed share of
    the causal pairs older than the local window) and density against the
    causal global mask ([P5] Step 2)."""
    mask = np.asarray(mask, dtype=bool)
    n = mask.shape[0]
    total_long = allowed_long = 0
    for i in range(n):
        for j in range(i + 1):
            if j < i - local_window + 1:
                total_long += 1
                allowed_long += int(mask[i, j])
    score = int(mask.sum())
    return {"visible_keys_mean": float(mask.sum(axis=1).mean()), "score_count": score,
            "long_range_coverage": allowed_long / total_long if total_long else 1.0,
            "density": score / (n * (n + 1) // 2)}


def block_mask_coverage(mask, n, bq, bk, causal, local_window):
    """``coverage_summary`` of the element-level mask of a block mask."""
    rows = np.arange(n) // bq
    cols = np.arange(n) // bk
    tok = np.asarray(mask, dtype=bool)[rows][:, cols]
    if causal:
        tok &= np.tril(np.ones((n, n), dtype=bool))
    return coverage_summary(tok, local_window)
