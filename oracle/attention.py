"""fp64 attention definitions: dense, restricted (masked) softmax, and the
tile-by-tile block-sparse online-softmax recurrence with the PV skip.

TEST INFRASTRUCTURE ONLY (see the package header): imported by tests, the
smoke check and the bench's CPU-baseline leg, never by the product path.

Pins (tests/test_oracle_attention.py):
* ``masked_attention`` -- the worked example of [P1] section 4 reproduces the
  printed union-mask MSEs, densities, max row error and bound; the 0.99/0.01
  counterexample of [P1] section 3.2; an all-ones mask equals dense attention.
* ``error_decomposition`` -- the exact identity and bound of [P1] section 3.2
  hold per row; brute force against a hand-expanded two-key case.
* ``block_sparse_attention`` -- with lambda = -inf it equals the restricted
  softmax of [P1] section 3.1 on the element-level mask of the kept blocks
  (a different code path: one dense masked softmax, no tiles); with lambda
  finite, a brute-force re-statement that drops exactly the skipped PV terms
  while keeping them in the normaliser ([P3] section 2.3).
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


def _as64(x):
    return np.asarray(x, dtype=np.float64)


def default_scale(d: int) -> float:
    """1/sqrt(d): the scaled dot product of [P1] section 3.1 and [P3] section 1."""
    return 1.0 / math.sqrt(d)


def softmax_rows(scores: np.ndarray) -> np.ndarray:
    """Row softmax with the row maximum subtracted first.

    A row whose every score is -inf has no defined softmax ([P1] section 3.1:
    an empty kept set is illegal), so such a row raises ``ValueError``.
    """
    scores = _as64(scores)
    row_max = scores.max(axis=-1, keepdims=True)
    if not np.all(np.isfinite(row_max)):
        raise ValueError("every query must keep at least one key")
    e = np.exp(scores - row_max)
    return e / e.sum(axis=-1, keepdims=True)


def masked_attention(q, k, v, mask, scale=None):
    """Attention restricted to the kept set S_i of each row ([P1] section 3.1).

    q: [Nq, d], k: [Nk, d], v: [Nk, dv]; mask: bool [Nq, Nk], True = key kept.
    Scores s_ij = q_i.k_j * scale (scale defaults to 1/sqrt(d)); dropped keys
    get -inf before the row softmax.  Returns (y, weights, lse) where lse is
    the natural-log log-sum-exp of the kept scores of each row.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    mask = np.asarray(mask, dtype=bool)
    if not mask.any(axis=-1).all():
        raise ValueError("every query must keep at least one key")
    if scale is None:
        scale = default_scale(q.shape[-1])
    s = (q @ k.T) * scale
    s = np.where(mask, s, NEG_INF)
    w = softmax_rows(s)
    m = s.max(axis=-1)
    lse = m + np.log(np.exp(s - m[:, None]).sum(axis=-1))
    return w @ v, w, lse


def dense_attention(q, k, v, causal=False, scale=None):
    """Full scaled-dot-product attention ([P1] section 3.1); with ``causal`` a
    key is visible iff its index is <= the query's ([P4] Step 2)."""
    nq, nk = q.shape[0], k.shape[0]
    if causal:
        mask = np.arange(nk)[None, :] <= np.arange(nq)[:, None]
    else:
        mask = np.ones((nq, nk), dtype=bool)
    y, _, lse = masked_attention(q, k, v, mask, scale)
    return y, lse


def error_decomposition(q, k, v, mask, scale=None):
    """The decomposition of [P1] section 3.2 for every row.

    Returns a dict with the full output y, the restricted output y_tilde
    (= r, the kept-set mean), the dropped-set mean u (NaN rows where nothing
    was dropped), the dropped mass alpha = 1 - z, and the bound 2*alpha*M with
    M the largest value norm.  The identity y_tilde - y = alpha * (r - u) is
    checked by the tests, not assumed here.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    mask = np.asarray(mask, dtype=bool)
    full = np.ones_like(mask)
    y, p, _ = masked_attention(q, k, v, full, scale)
    y_t, _, _ = masked_attention(q, k, v, mask, scale)
    z = (p * mask).sum(axis=-1)
    alpha = 1.0 - z
    dropped = p * (~mask)
    with np.errstate(invalid="ignore", divide="ignore"):
        u = (dropped @ v) / dropped.sum(axis=-1, keepdims=True)
    m_norm = np.linalg.norm(v, axis=-1).max()
    return {"y": y, "y_tilde": y_t, "r": y_t, "u": u, "alpha": alpha,
            "z": z, "bound": 2.0 * alpha * m_norm, "p": p}


def kept_blocks_to_token_mask(kept, n, bq, bk, causal=False):
    """Element-level mask of a block mask M_g ([P3] section 2.1; [P4] Step 4):
    a kept (q-block, k-block) pair opens every (i, j) in it, then causality
    (j <= i) is applied element by element."""
    kept = np.asarray(kept, dtype=bool)
    rows = np.arange(n) // bq
    cols = np.arange(n) // bk
    mask = kept[rows][:, cols]
    if causal:
        mask &= np.arange(n)[None, :] <= np.arange(n)[:, None]
    return mask


def block_sparse_attention(q, k, v, kept, bq, bk, causal=False, lam=NEG_INF,
                           scale=None, qblocks=None, skip_override=None,
                           band=1e-3):
    """Sparse FlashAttention forward of [P3] sections 2.1 and 2.3, one head.

    q, k: [N, d]; v: [N, dv]; kept: bool [nQB, nKB] (M_g).  For every
    q-block (all, or those listed in ``qblocks``) the kept k-blocks are
    visited in ascending order.  Per tile:

      S       = Q_i K_j^T * scale, with -inf where j > i (causal) -- tail
                rows/columns past N simply do not exist;
      m_local = rowmax(S);  m_new = max(m_old, m_local)
      P       = exp(S - m_new)
      l       = exp(m_old - m_new) * l + rowsum(P)
      gap     = max over the q-block's rows of (m_local - m_new), rows whose
                m_local is -inf excluded (they hold no score in this tile)
      if gap < lam:  skip P V (O unchanged; the scale factor is 1 because
                     every row's maximum did not move)
      else:          O = exp(m_old - m_new) * O + P V

    and at the end out = O / l, lse = m + ln l.  The skip group is the whole
    q-block (one decision per tile).  Strict ``<`` skips; equality computes.

    ``skip_override`` maps (qb, kb) -> bool and replaces the oracle's own
    decision only where |gap - lam| <= band (a decision on the boundary, where
    both answers are correct); an override elsewhere raises ValueError.

    Returns dict(out [N, dv] (rows of unvisited q-blocks are NaN),
    lse [N], skips {(qb, kb): bool}, gaps {(qb, kb): float}).
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    kept = np.asarray(kept, dtype=bool)
    n, d = q.shape
    dv = v.shape[1]
    if scale is None:
        scale = default_scale(d)
    nqb = -(-n // bq)
    nkb = -(-n // bk)
    if kept.shape != (nqb, nkb):
        raise ValueError(f"mask shape {kept.shape} != {(nqb, nkb)}")
    out = np.full((n, dv), np.nan)
    lse = np.full(n, np.nan)
    skips, gaps = {}, {}
    todo = range(nqb) if qblocks is None else qblocks
    for qb in todo:
        i0, i1 = qb * bq, min(n, (qb + 1) * bq)
        rows = np.arange(i0, i1)
        m = np.full(i1 - i0, NEG_INF)
        l = np.zeros(i1 - i0)
        o = np.zeros((i1 - i0, dv))
        for kb in np.flatnonzero(kept[qb]):
            j0, j1 = kb * bk, min(n, (kb + 1) * bk)
            s = (q[i0:i1] @ k[j0:j1].T) * scale
            if causal:
                s = np.where(np.arange(j0, j1)[None, :] <= rows[:, None], s, NEG_INF)
            m_local = s.max(axis=1)
            m_new = np.maximum(m, m_local)
            live = np.isfinite(m_new)
            p = np.zeros_like(s)
            p[live] = np.exp(s[live] - m_new[live, None])
            corr = np.ones_like(m)
            has_old = live & np.isfinite(m)
            corr[live & ~np.isfinite(m)] = 0.0
            corr[has_old] = np.exp(m[has_old] - m_new[has_old])
            l = corr * l + p.sum(axis=1)
            row_gap = np.where(np.isfinite(m_local), m_local - np.where(live, m_new, 0.0), NEG_INF)
            gap = float(row_gap.max())
            skip = bool(gap < lam)
            if skip_override is not None and (qb, int(kb)) in skip_override:
                forced = bool(skip_override[(qb, int(kb))])
                if forced != skip:
                    if not (abs(gap - lam) <= band):
                        raise ValueError(f"override of tile {(qb, int(kb))} off the lambda band: gap={gap}")
                    skip = forced
            if not skip:
                o = corr[:, None] * o + p @ v[j0:j1]
            skips[(qb, int(kb))] = skip
            gaps[(qb, int(kb))] = gap
            m = m_new
        if not np.all(l > 0):
            raise ValueError(f"q-block {qb} has a query row with no visible key")
        out[i0:i1] = o / l[:, None]
        lse[i0:i1] = m + np.log(l)
    return {"out": out, "lse": lse, "skips": skips, "gaps": gaps}


def block_sparse_attention_heads(q, k, v, kept, bq, bk, causal=False,
                                 lam=NEG_INF, scale=None, heads=None,
                                 qblocks=None, skip_override=None, band=1e-3):
    """``block_sparse_attention`` over BNSD tensors.

    q: [B, Hq, N, d]; k, v: [B, Hkv, N, d/dv]; kept: [B, Hq, nQB, nKB].
    Query head h reads kv head h // (Hq // Hkv) (grouped-query attention;
    not on the pages -- the plain reading of sharing one K/V among a group).
    ``heads``: optional list of (b, h) pairs; ``skip_override`` maps
    (b, h, qb, kb) -> bool.  Returns out/lse arrays (NaN where not computed)
    and skips/gaps keyed by (b, h, qb, kb).
    """
    B, Hq, N, _ = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    out = np.full(q.shape[:3] + (v.shape[3],), np.nan)
    lse = np.full(q.shape[:3], np.nan)
    skips, gaps = {}, {}
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        ov = None
        if skip_override is not None:
            ov = {(qb, kb): s for (bb, hh, qb, kb), s in skip_override.items() if bb == b and hh == h}
        r = block_sparse_attention(q[b, h], k[b, h // group], v[b, h // group], kept[b, h],
                                   bq, bk, causal, lam, scale, qblocks, ov, band)
        out[b, h] = r["out"]
        lse[b, h] = r["lse"]
        for key, val in r["skips"].items():
            skips[(b, h) + key] = val
            gaps[(b, h) + key] = r["gaps"][key]
    return {"out": out, "lse": lse, "skips": skips, "gaps": gaps}


def dropped_mass_from_lse(lse_sparse, lse_dense):
    """Per-row dropped probability mass alpha = 1 - z with
    z = exp(lse_kept - lse_full) ([P1] section 3.2: z is the kept mass)."""
    return 1.0 - np.exp(_as64(lse_sparse) - _as64(lse_dense))
