"""Bisect TopCdf's tau so the oracle's block mask reaches a target sparsity.

Run as ``python -m oracle.tune_tau <workload> [target [theta]]``.  It generates the
workload's seeded inputs, applies the workload's layout, runs the oracle's
mask prediction once, and bisects tau on the oracle's own c_excl values
(the kept set of TopCdf at tau is {c_excl < tau}), 40 steps or until the
block sparsity is within 0.005 of the target.  Sparsity is the skipped
fraction of the causally valid block products summed over batch and heads
(the "sparsity" of the SpargeAttention notes, section 3.2).  The printed tau
is what ``long_context_mean_b200/inputs.py`` freezes for that workload; no
value produced by the CUDA library is read.
"""

from __future__ import annotations

import sys

import numpy as np

from . import layout as Y
from . import predict as Pr


def oracle_parts(w, batches=None, heads=None):
    from long_context_mean_b200 import inputs as I   # seeded generators only
    g = I.gen_qkv(w, heads=heads, batches=batches)
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    q = Y.reorder(g["q"], perm)
    k = Y.reorder(g["k"], perm)
    return Pr.predict_mask(q, k, w.bq, w.bk, w.tau, w.theta, w.causal, w.sink_tokens,
                           w.txt_len, w.local_window, w.anchor_tokens)


def sparsity_at(parts, tau):
    top = np.nan_to_num(parts["c_excl"], nan=np.inf) < tau
    mask = (top & parts["valid"][:, None]) | parts["forced"]
    return Pr.block_sparsity(mask, np.broadcast_to(parts["valid"][:, None], mask.shape))


def bisect_tau(parts, target, steps=40, tol=0.005):
    lo, hi = 0.0, 1.0          # sparsity falls as tau grows
    tau = 0.5
    for _ in range(steps):
        tau = 0.5 * (lo + hi)
        s = sparsity_at(parts, tau)
        if abs(s - target) <= tol:
            break
        if s > target:
            lo = tau
        else:
            hi = tau
    return tau, sparsity_at(parts, tau)


def main(argv):
    from long_context_mean_b200 import inputs as I
    w = I.WORKLOADS[argv[0]]
    target = float(argv[1]) if len(argv) > 1 else w.target_sparsity
    if len(argv) > 2:                     # optional theta override for sweeps
        w = w.with_(theta=float(argv[2]))
    parts = oracle_parts(w)
    floor = Pr.block_sparsity(parts["forced"], np.broadcast_to(parts["valid"][:, None], parts["forced"].shape))
    tau, s = bisect_tau(parts, target)
    print(f"{w.name}: theta={w.theta} forced-only sparsity={floor:.4f} "
          f"target={target} tau={tau:.6f} sparsity={s:.4f}")


if __name__ == "__main__":
    main(sys.argv[1:])
