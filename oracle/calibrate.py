"""fp64 per-layer calibration of (tau, theta) and then lambda, as the
SpargeAttention notes describe it ([P3] section 2.4).

TEST INFRASTRUCTURE ONLY (see the package header).

The notes search, per attention layer, first (tau, theta) so that the
relative L1 error of the output stays below l1 while the sparsity is as
large as possible, then lambda so that the total error stays below l2:

    L1 = sum |O - O'| / sum |O|     (O dense, O' sparse)

Readings where the notes are silent (no grid, no tie rule, no sparsity
measure for lambda is printed):
  * the search is exhaustive over caller-given grids, which should contain
    tau = 1 with theta <= 0 (every eligible block kept) and lambda = -inf, so
    that a feasible point always exists;
  * step 1 maximises block sparsity (1 - kept / causally valid tiles);
    step 2 maximises the skipped fraction of the kept tiles' P V products;
  * a point is feasible when its L1 is strictly below the bound;
  * ties: the smaller L1 wins, then the larger tau, the smaller theta, the
    larger lambda (the grid order decides nothing).

Pins (tests/test_oracle_calibrate.py): relative L1 on closed-form arrays; the
selection rule on hand-made tables; on a small problem the full-mask point
(tau = 1, theta = 0) has L1 = 0 up to rounding (< 1e-12), and the chosen point is feasible
and at least as sparse as every other feasible point found by brute force.
"""

from __future__ import annotations

import math

import numpy as np

from . import attention as A
from . import predict as Pr


def relative_l1(ref, x) -> float:
    """sum |ref - x| / sum |ref| in float64 ([P3] section 2.4)."""
    ref = np.asarray(ref, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    den = np.abs(ref).sum()
    return float(np.abs(ref - x).sum() / den) if den > 0 else 0.0


def select_tau_theta(rows, l1):
    """rows: dicts with tau, theta, l1, sparsity.  The feasible (l1 < bound)
    row of largest sparsity; ties by smaller l1, larger tau, smaller theta."""
    feas = [r for r in rows if r["l1"] < l1]
    if not feas:
        return None
    return min(feas, key=lambda r: (-r["sparsity"], r["l1"], -r["tau"], r["theta"]))


def select_lambda(rows, l2):
    """rows: dicts with lam, l1, pv_skip.  The feasible (l1 < bound) row of
    largest skipped PV fraction; ties by smaller l1, then larger lambda."""
    feas = [r for r in rows if r["l1"] < l2]
    if not feas:
        return None
    return min(feas, key=lambda r: (-r["pv_skip"], r["l1"], -r["lam"]))


def valid_tiles(n, bq, bk, causal):
    """Causally valid (q-block, k-block) pairs of one head."""
    nqb, nkb = -(-n // bq), -(-n // bk)
    if not causal:
        return nqb * nkb
    return sum(sum(1 for kb in range(nkb) if not Pr.causal_future(qb, kb, n, bq, bk)) for qb in range(nqb))


def calibrate(q, k, v, bq, bk, taus, thetas, lams, l1, l2, causal=False, sink_tokens=0,
              txt_len=0, local_window=0, anchor_tokens=0):
    """q [B, Hq, N, d], k/v [B, Hkv, N, d] (already in the layout's order).
    Returns dict(tau, theta, lam, step1 rows, step2 rows)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, Hq, N, _ = q.shape
    group = Hq // k.shape[1]
    dense = np.stack([np.stack([A.dense_attention(q[b, h], k[b, h // group], v[b, h // group], causal)[0]
                                for h in range(Hq)]) for b in range(B)])
    total_valid = B * Hq * valid_tiles(N, bq, bk, causal)
    step1 = []
    masks = {}
    for tau in taus:
        for theta in thetas:
            pm = Pr.predict_mask(q, k, bq, bk, tau, theta, causal, sink_tokens, txt_len, local_window,
                                 anchor_tokens)
            mask = pm["mask"]
            r = A.block_sparse_attention_heads(q, k, v, mask, bq, bk, causal)
            step1.append({"tau": float(tau), "theta": float(theta), "l1": relative_l1(dense, r["out"]),
                          "sparsity": 1.0 - mask.sum() / total_valid})
            masks[(float(tau), float(theta))] = mask
    best = select_tau_theta(step1, l1)
    if best is None:
        raise ValueError("no (tau, theta) point meets the L1 bound; add tau = 1, theta = 0 to the grid")
    mask = masks[(best["tau"], best["theta"])]
    kept = int(mask.sum())
    step2 = []
    for lam in lams:
        r = A.block_sparse_attention_heads(q, k, v, mask, bq, bk, causal, lam=lam)
        step2.append({"lam": float(lam), "l1": relative_l1(dense, r["out"]),
                      "pv_skip": sum(r["skips"].values()) / kept if kept else 0.0})
    lam_best = select_lambda(step2, l2)
    if lam_best is None:
        raise ValueError("no lambda meets the L1 bound; add lambda = -inf to the grid")
    return {"tau": best["tau"], "theta": best["theta"], "lam": lam_best["lam"], "step1": step1,
            "step2": step2}
