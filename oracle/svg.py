"""fp64 per-head choice between a spatial and a temporal mask, and the
attention it leads to: the Sparse VideoGen comparison of [P1] ("AIGC
基本功｜视频稀疏注意力的误差与布局", sections 3.3, 3.4, 4 and 5).

TEST INFRASTRUCTURE ONLY (see the package header).

What the page fixes:
  * section 3.3: on a frame-major grid (token t*P + p, P = H*W) the spatial
    mask keeps the pairs of one frame, the temporal mask the pairs of one
    position across frames;
  * section 3.4: permuting Q, K, V and both mask axes together permutes the
    output rows and nothing else;
  * section 4: a tile is computed whole once it holds one allowed pair (the
    block ledger), and grouping a position's frames together turns the
    temporal mask's scattered pairs into whole tiles;
  * section 5: the online profile samples query rows, computes dense
    attention and both candidates there, compares them by the mean squared
    error of the outputs and takes the argmin per head; the temporal heads'
    video tokens go from frame-major to token-major order while trailing
    context tokens keep their place.

Readings where the page is silent:
  * text tokens (the ``txt_len`` tokens after the video tokens) pair with
    every token in both candidates (the page leaves context tokens to the
    models and only keeps them in place in the layout);
  * the candidates run at block granularity: the kept tiles are the block
    cover of the element mask (the section 4 ledger), and the block-sparse
    recurrence sees every key of a kept tile; on tiles aligned with frames
    (spatial) or positions (temporal) the cover is the element mask itself;
  * the MSE of a head averages the squared error over the sampled rows'
    outputs, a row drawn twice counting twice (the page notes sampling with
    replacement); a tie goes to the spatial candidate.

Pins (tests/test_oracle_svg.py): the 4096 / 1024 / 256 pair counts and the
64 -> 16 tile ledger of section 4 (golden fixture); the block cover against
the closed-form interval rule on random grids; on aligned tiles each
candidate equals the element-masked softmax of section 3.1 (a different
code path), the temporal one through the permutation of section 3.4; on the
worked example of section 4 the choice is [spatial, temporal], as section 5
reports, and a head on the wrong candidate is worse by orders of magnitude.
"""

from __future__ import annotations

import numpy as np

from . import attention as A

SPATIAL, TEMPORAL = 0, 1


def element_mask_rows(T: int, H: int, W: int, txt_len: int, kind: int, rows) -> np.ndarray:
    """Rows ``rows`` (original token indices) of the element mask: bool
    [len(rows), N] over the frame-major order, N = T*H*W + txt_len."""
    P = H * W
    nv = T * P
    n = nv + txt_len
    rows = np.asarray(rows, dtype=np.int64)
    group = np.full(n, -1, dtype=np.int64)           # -1: a text token
    group[:nv] = np.repeat(np.arange(T), P) if kind == SPATIAL else np.tile(np.arange(P), T)
    gr = group[rows]
    return (gr[:, None] == group[None, :]) | (gr[:, None] < 0) | (group[None, :] < 0)


def element_mask(T: int, H: int, W: int, txt_len: int, kind: int) -> np.ndarray:
    """bool [N, N] over the frame-major order, N = T*H*W + txt_len."""
    return element_mask_rows(T, H, W, txt_len, kind, np.arange(T * H * W + txt_len))


def token_major_perm(T: int, H: int, W: int, txt_len: int) -> np.ndarray:
    """perm[n] = frame-major source of token-major position n: the video
    part is regrouped by position (position p's frames at p*T .. p*T+T-1),
    the text tail stays in place (section 5)."""
    P = H * W
    nv = T * P
    pixel = np.tile(np.arange(P), T)
    video = np.argsort(pixel, kind="stable")
    return np.concatenate([video, np.arange(nv, nv + txt_len)]).astype(np.int64)


def block_cover(mask: np.ndarray, bq: int, bk: int) -> np.ndarray:
    """Tile (qb, kb) is kept iff it holds one allowed pair (section 4)."""
    n = mask.shape[0]
    nqb, nkb = -(-n // bq), -(-n // bk)
    kept = np.zeros((nqb, nkb), dtype=bool)
    for qb in range(nqb):
        for kb in range(nkb):
            kept[qb, kb] = mask[qb * bq:(qb + 1) * bq, kb * bk:(kb + 1) * bk].any()
    return kept


def candidate_order(T, H, W, txt_len, kind) -> np.ndarray:
    """The token order a candidate runs in: identity (spatial) or token-major (temporal)."""
    n = T * H * W + txt_len
    return np.arange(n) if kind == SPATIAL else token_major_perm(T, H, W, txt_len)


def head_block_mask(T, H, W, txt_len, kind, bq, bk) -> np.ndarray:
    """The kept tiles of a candidate in its own order: the block cover of
    Pi A Pi^T (section 3.4) for the candidate's order Pi."""
    perm = candidate_order(T, H, W, txt_len, kind)
    m = element_mask(T, H, W, txt_len, kind)
    return block_cover(m[np.ix_(perm, perm)], bq, bk)


def candidate_attention(q, k, v, T, H, W, txt_len, kind, bq, bk, kept=None):
    """One head's output and lse under a candidate, back in the original
    order: permute, run the tiles, put the rows back (section 3.4)."""
    perm = candidate_order(T, H, W, txt_len, kind)
    if kept is None:
        kept = head_block_mask(T, H, W, txt_len, kind, bq, bk)
    r = A.block_sparse_attention(np.asarray(q)[perm], np.asarray(k)[perm], np.asarray(v)[perm], kept, bq, bk)
    out = np.empty_like(r["out"])
    lse = np.empty_like(r["lse"])
    out[perm] = r["out"]
    lse[perm] = r["lse"]
    return out, lse


def sampled_mse(ref, x, rows) -> float:
    """Mean of (ref - x)^2 over the sampled rows' outputs (section 5)."""
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size == 0:
        return 0.0
    d = np.asarray(ref, dtype=np.float64)[rows] - np.asarray(x, dtype=np.float64)[rows]
    return float(np.mean(d * d))


def select_heads(q, k, v, T, H, W, txt_len, bq, bk, rows):
    """q, k, v: [BH, N, d] (one K/V per query head).  Returns (choice [BH],
    mse [2, BH]): per head the MSE of each candidate against dense
    attention on the sampled rows and the argmin (ties to spatial)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    BH = q.shape[0]
    kept = [head_block_mask(T, H, W, txt_len, c, bq, bk) for c in (SPATIAL, TEMPORAL)]
    mse = np.zeros((2, BH))
    for h in range(BH):
        dense = A.dense_attention(q[h], k[h], v[h])[0]
        for c in (SPATIAL, TEMPORAL):
            out, _ = candidate_attention(q[h], k[h], v[h], T, H, W, txt_len, c, bq, bk, kept[c])
            mse[c, h] = sampled_mse(dense, out, rows)
    choice = np.where(mse[TEMPORAL] < mse[SPATIAL], TEMPORAL, SPATIAL)
    return choice, mse


def svg_attention(q, k, v, choice, T, H, W, txt_len, bq, bk):
    """Each head under its chosen candidate; q, k, v [BH, N, d].  Returns
    (out [BH, N, dv], lse [BH, N]) in the original order."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    kept = [head_block_mask(T, H, W, txt_len, c, bq, bk) for c in (SPATIAL, TEMPORAL)]
    out = np.empty(q.shape[:2] + (v.shape[2],))
    lse = np.empty(q.shape[:2])
    for h in range(q.shape[0]):
        c = int(choice[h])
        out[h], lse[h] = candidate_attention(q[h], k[h], v[h], T, H, W, txt_len, c, bq, bk, kept[c])
    return out, lse
