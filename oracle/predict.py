"""fp64 mask prediction: block pooling, the intra-block similarity guard,
compressed softmax with TopCdf, forced rows/columns, block mask, CSR lists.

TEST INFRASTRUCTURE ONLY (see the package header).

Pipeline ([P3] section 2.2, with [P2] rf_v2 / ada_bsa and [P5] anchors):
  1. q_hat = mean of each query block, k_hat = mean of each key block, over
     the tokens the block really holds (a ragged tail block uses its count).
  2. s = mean pairwise cosine similarity of the block's tokens (diagonal
     included), computed here by brute force over all pairs.
  3. S_hat = q_hat k_hat^T / sqrt(d); key blocks with s_k < theta, and
     causally-future key blocks, get -inf; row softmax.
  4. TopCdf(tau): sort the row by probability descending (ties: lower block
     index first) and keep a block iff the cumulative mass *before* it is
     < tau * (row total).
  5. Forced full rows where s_q < theta, forced full columns where
     s_k < theta; sink tokens (front) and text tokens (back) force their
     rows and columns; anchor tokens (front) force their columns; a
     block-level local window keeps every block pair holding some (i, j)
     with 0 <= i - j < w; everything is then ANDed with causal validity.
  6. CSR lists (column indices ascending) and a work order (rows by
     descending kept count, ties by ascending row index, optionally inside
     groups of consecutive heads: a scheduling choice of this library).

Readings where the pages are silent or garbled:
  * CosSim: the notes print mean(X X^T / |max(X X^T)|) while naming it a
    cosine similarity; the standard mean pairwise cosine (x_hat = x/|x|,
    zero vectors contribute 0) is used.  ``cossim_literal`` keeps the printed
    form as a diagnostic only.
  * theta compares with strict '<'; theta <= 0 disables the guard.
  * S_hat includes 1/sqrt(d).
  * TopCdf keeps the element that crosses tau (the prose: "reach tau"), not
    the printed ``cumsum <= tau*sum`` (which can keep nothing).
  * A row whose every entry is -inf selects nothing by TopCdf (its blocks
    are then covered by the forced columns).
  * TopCdf runs over all eligible blocks; forced blocks are ORed afterwards.
  * Causal block validity: k-block kb is future for q-block qb iff
    kb*bk > (last row of qb).
  * Grouped-query attention: query head h uses kv head h // (Hq/Hkv).

Pins (tests/test_oracle_predict.py): CosSim brute force equals the closed
form |sum x_hat|^2 / n^2, identical tokens give 1, n orthonormal tokens give
1/n; TopCdf keeps {0.6, 0.3} of [0.6, 0.3, 0.1] at tau = 0.8 (the notes'
teaching example), keeps only the arg-max as tau -> 0+, keeps every p > 0 at
tau = 1, and equals an exhaustive smallest-prefix search on random rows;
the local window / anchor masks reproduce the unit tests printed on [P4]
and [P5]; the block-level window is checked against brute force over
element pairs.
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


def n_blocks(n: int, b: int) -> int:
    return -(-n // b)


def block_ranges(n: int, b: int):
    return [(i * b, min(n, (i + 1) * b)) for i in range(n_blocks(n, b))]


def pool_blocks(x, b):
    """Block means over the true token count ([P3] section 2.2 step 1)."""
    x = np.asarray(x, dtype=np.float64)
    return np.stack([x[s:e].mean(axis=0) for s, e in block_ranges(x.shape[0], b)])


def unit_rows(x):
    x = np.asarray(x, dtype=np.float64)
    nrm = np.linalg.norm(x, axis=-1, keepdims=True)
    out = np.zeros_like(x)
    np.divide(x, nrm, out=out, where=nrm > 0)
    return out


def cossim_block(xb):
    """Mean pairwise cosine of one block's tokens, all n^2 ordered pairs."""
    u = unit_rows(xb)
    return float((u @ u.T).mean())


def cossim_blocks(x, b):
    x = np.asarray(x, dtype=np.float64)
    return np.array([cossim_block(x[s:e]) for s, e in block_ranges(x.shape[0], b)])


def cossim_literal(xb):
    """Diagnostic only: the printed form mean(X X^T / |max(X X^T)|)."""
    g = np.asarray(xb, dtype=np.float64) @ np.asarray(xb, dtype=np.float64).T
    return float((g / abs(g.max())).mean())


def causal_future(qb, kb, n, bq, bk):
    last_row = min(n, (qb + 1) * bq) - 1
    return kb * bk > last_row


def topcdf(p, tau):
    """TopCdf(tau) over one row of probabilities ([P3] section 2.2).

    Returns (kept bool array, c_excl) where c_excl is each entry's
    exclusive cumulative mass in the sorted order divided by the row total
    (the quantity compared with tau).  Zero-probability entries (the -inf
    scores) are never kept when tau <= 1.
    """
    p = np.asarray(p, dtype=np.float64)
    idx = np.arange(p.size)
    order = np.lexsort((idx, -p))
    ps = p[order]
    incl = np.cumsum(ps)
    total = incl[-1] if p.size else 0.0
    excl = incl - ps
    kept = np.zeros(p.size, dtype=bool)
    c = np.full(p.size, np.nan)
    if total > 0:
        kept[order] = excl < tau * total
        c[order] = excl / total
    return kept, c


def compressed_probs(qhat_row, khat, eligible, d):
    """Softmax over the eligible entries of q_hat k_hat^T / sqrt(d); zeros
    elsewhere; all zeros if nothing is eligible."""
    s = (khat @ np.asarray(qhat_row, dtype=np.float64)) / math.sqrt(d)
    p = np.zeros(khat.shape[0])
    if eligible.any():
        se = s[eligible]
        e = np.exp(se - se.max())
        p[eligible] = e / e.sum()
    return p


def predict_mask_batch(q, k, bq, bk, tau, theta, causal=False, sink_tokens=0,
                       txt_len=0, local_window=0, anchor_tokens=0):
    """Block mask for one batch element.

    q: [Hq, N, d]; k: [Hkv, N, d].  Returns a dict with
      mask [Hq, nQB, nKB] bool (the final M_g), top [Hq, nQB, nKB] (TopCdf
      picks alone), forced [Hq, nQB, nKB] (the tau-independent part), c_excl [Hq, nQB, nKB] (NaN where not eligible),
      s_q [Hq, nQB], s_k [Hkv, nKB], qhat [Hq, nQB, d], khat [Hkv, nKB, d],
      forced_rows [Hq, nQB], forced_cols [Hkv, nKB], valid [nQB, nKB].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    Hq, N, d = q.shape
    Hkv = k.shape[0]
    group = Hq // Hkv
    nqb, nkb = n_blocks(N, bq), n_blocks(N, bk)
    qhat = np.stack([pool_blocks(q[h], bq) for h in range(Hq)])
    khat = np.stack([pool_blocks(k[g], bk) for g in range(Hkv)])
    s_q = np.stack([cossim_blocks(q[h], bq) for h in range(Hq)])
    s_k = np.stack([cossim_blocks(k[g], bk) for g in range(Hkv)])
    guard = theta > 0
    low_q = (s_q < theta) if guard else np.zeros_like(s_q, dtype=bool)
    low_k = (s_k < theta) if guard else np.zeros_like(s_k, dtype=bool)

    valid = np.ones((nqb, nkb), dtype=bool)
    if causal:
        for qb in range(nqb):
            for kb in range(nkb):
                valid[qb, kb] = not causal_future(qb, kb, N, bq, bk)

    # Structural forced rows/columns: sink at the front, text at the back,
    # anchors (keys only) at the front.
    row_struct = np.zeros(nqb, dtype=bool)
    col_struct = np.zeros(nkb, dtype=bool)
    for qb, (s, e) in enumerate(block_ranges(N, bq)):
        if s < sink_tokens or (txt_len > 0 and e - 1 >= N - txt_len):
            row_struct[qb] = True
    for kb, (s, e) in enumerate(block_ranges(N, bk)):
        if s < sink_tokens or s < anchor_tokens or (txt_len > 0 and e - 1 >= N - txt_len):
            col_struct[kb] = True

    window = np.zeros((nqb, nkb), dtype=bool)
    if local_window > 0:
        for qb, (i0, i1) in enumerate(block_ranges(N, bq)):
            for kb, (j0, j1) in enumerate(block_ranges(N, bk)):
                window[qb, kb] = (i1 - 1 >= j0) and (i0 - (j1 - 1) < local_window)

    top = np.zeros((Hq, nqb, nkb), dtype=bool)
    c_excl = np.full((Hq, nqb, nkb), np.nan)
    mask = np.zeros((Hq, nqb, nkb), dtype=bool)
    forced = np.zeros((Hq, nqb, nkb), dtype=bool)
    for h in range(Hq):
        g = h // group
        for qb in range(nqb):
            eligible = valid[qb] & ~low_k[g]
            p = compressed_probs(qhat[h, qb], khat[g], eligible, d)
            if eligible.any():
                kept, c = topcdf(p, tau)
                kept &= eligible
                top[h, qb] = kept
                c_excl[h, qb, eligible] = c[eligible]
        rows = low_q[h] | row_struct
        cols = low_k[g] | col_struct
        forced[h] = (rows[:, None] | cols[None, :] | window) & valid
        mask[h] = top[h] & valid | forced[h]
    return {"mask": mask, "top": top, "forced": forced, "c_excl": c_excl, "s_q": s_q, "s_k": s_k,
            "qhat": qhat, "khat": khat, "forced_rows": low_q | row_struct[None, :],
            "forced_cols": low_k | col_struct[None, :], "valid": valid}


def predict_mask(q, k, bq, bk, tau, theta, causal=False, sink_tokens=0,
                 txt_len=0, local_window=0, anchor_tokens=0):
    """``predict_mask_batch`` over a batch: q [B, Hq, N, d], k [B, Hkv, N, d];
    every returned array gains a leading B axis."""
    parts = [predict_mask_batch(q[b], k[b], bq, bk, tau, theta, causal, sink_tokens,
                                txt_len, local_window, anchor_tokens) for b in range(q.shape[0])]
    return {key: np.stack([p[key] for p in parts]) for key in parts[0]}


def empty_rows(mask, n, bq, bk, causal):
    """Element-level check that every query row keeps a visible key
    ([P1] section 3.1: an empty kept set is illegal).  mask: [..., nQB, nKB].
    Returns a bool array [..., nQB], True where some row of the q-block
    would see no key."""
    mask = np.asarray(mask, dtype=bool)
    nqb, nkb = mask.shape[-2:]
    bad = np.zeros(mask.shape[:-1], dtype=bool)
    for qb in range(nqb):
        first_row = qb * bq
        if causal:
            ok_cols = np.arange(nkb) * bk <= first_row
            bad[..., qb] = ~(mask[..., qb, :] & ok_cols).any(axis=-1)
        else:
            bad[..., qb] = ~mask[..., qb, :].any(axis=-1)
    return bad


def mask_to_csr(mask, order_group=0):
    """CSR form of a block mask [..., nQB, nKB] flattened over its leading axes
    in row-major order: row_ptr [R+1], col_idx ascending within a row, the
    work order, and the kept total.  The work order (a scheduling choice of
    this library, not the pages'): rows by descending count, ties by
    ascending row index; with order_group = g > 0, the rows first form groups
    of g consecutive heads (g * nQB rows each, the groups in order) and that
    order applies inside each group."""
    mask = np.asarray(mask, dtype=bool)
    nqb, nkb = mask.shape[-2], mask.shape[-1]
    flat = mask.reshape(-1, nkb)
    counts = flat.sum(axis=1).astype(np.int64)
    row_ptr = np.zeros(flat.shape[0] + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.concatenate([np.flatnonzero(r) for r in flat]) if flat.size else np.zeros(0, np.int64)
    rows = np.arange(flat.shape[0])
    group = rows // (order_group * nqb) if order_group > 0 else np.zeros_like(rows)
    order = np.lexsort((rows, -counts, group))
    return {"row_ptr": row_ptr, "col_idx": col_idx.astype(np.int64), "order": order,
            "counts": counts, "kept_total": int(counts.sum())}


def block_sparsity(mask, valid):
    """Skipped fraction of the valid block products ([P3] section 3.2:
    sparsity counts skipped block multiplications)."""
    mask = np.asarray(mask, dtype=bool)
    valid = np.broadcast_to(np.asarray(valid, dtype=bool), mask.shape)
    return 1.0 - mask.sum() / valid.sum()
