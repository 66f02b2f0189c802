"""Per-layer calibration of (tau, theta) and then lambda on the GPU, as the
SpargeAttention notes describe it ([P3] section 2.4): choose (tau, theta)
with the largest block sparsity whose relative L1 output error
sum |O - O'| / sum |O| against dense attention stays below l1, then the
lambda with the largest skipped fraction of P V products whose error stays
below l2.

Every output and every error sum comes from the library's kernels (the
block-sparse path, ``sa_dense_attn`` and ``sa_l1_error``); this module only
walks the grids.  Readings where the notes are silent: the grids are the
caller's (they should hold tau = 1 with theta <= 0, and lambda = -inf, so a
feasible point exists); a point is feasible when its error is strictly below
the bound; ties go to the smaller error, then the larger tau, the smaller
theta, the larger lambda.
"""

from __future__ import annotations

import math

from . import sa


def _valid_tiles(N, bq, bk, causal):
    nqb, nkb = -(-N // bq), -(-N // bk)
    if not causal:
        return nqb * nkb
    return sum(min(nkb, (min(N, (qb + 1) * bq) - 1) // bk + 1) for qb in range(nqb))


def calibrate(w, q, k, v, taus, thetas, lams, l1, l2, device="cuda"):
    """w: a workload description (shape, layout, block sizes and the forced
    structure of ``inputs.Workload``); q, k, v: BNSD device tensors in the
    original token order.  Returns dict(tau, theta, lam, step1, step2)."""
    import torch
    pipe = sa.pipeline_for(w, device=device, log_skips=True)
    shape = sa.Shape(w.B, w.Hq, w.Hkv, w.N, w.d, w.dv, sa.dtype_code(q), 0)
    dense = torch.empty_like(pipe.out)
    dense_lse = torch.empty_like(pipe.lse)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    sa.dense_attn(q, k, v, shape, w.causal, 0.0, dense, dense_lse, st)
    if sa.read_status(st) != sa.SA_OK:
        raise RuntimeError("dense attention reported an error")
    sums = torch.zeros(2, dtype=torch.float64, device=device)
    total_valid = w.B * w.Hq * _valid_tiles(w.N, w.bq, w.bk, w.causal)

    def run(tau, theta, lam):
        pipe.params.tau, pipe.params.theta, pipe.lam = float(tau), float(theta), float(lam)
        out, _ = pipe.run(q, k, v)
        sa.l1_error(dense, out, sums)
        if pipe.status() != sa.SA_OK:
            raise RuntimeError(f"device status {pipe.status()} at tau={tau} theta={theta} lam={lam}")
        s = sums.cpu().tolist()
        kept = int(pipe.mask.kept_total.item())
        err = s[0] / s[1] if s[1] > 0 else 0.0
        return err, kept

    step1 = []
    for tau in taus:
        for theta in thetas:
            err, kept = run(tau, theta, -math.inf)
            step1.append({"tau": float(tau), "theta": float(theta), "l1": err,
                          "sparsity": 1.0 - kept / total_valid})
    feas = [r for r in step1 if r["l1"] < l1]
    if not feas:
        raise ValueError("no (tau, theta) point meets the L1 bound; add tau = 1, theta = 0 to the grid")
    best = min(feas, key=lambda r: (-r["sparsity"], r["l1"], -r["tau"], r["theta"]))
    step2 = []
    for lam in lams:
        err, kept = run(best["tau"], best["theta"], lam)
        skipped = int(pipe.skip_log[:kept].cpu().numpy().sum()) if kept else 0
        step2.append({"lam": float(lam), "l1": err, "pv_skip": skipped / kept if kept else 0.0})
    feas2 = [r for r in step2 if r["l1"] < l2]
    if not feas2:
        raise ValueError("no lambda meets the L1 bound; add lambda = -inf to the grid")
    lam_best = min(feas2, key=lambda r: (-r["pv_skip"], r["l1"], -r["lam"]))
    return {"tau": best["tau"], "theta": best["theta"], "lam": lam_best["lam"], "step1": step1, "step2": step2}
