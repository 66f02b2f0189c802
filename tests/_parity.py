"""Helpers shared by the GPU parity tests: run the CUDA path through the C
ABI binding and the fp64 oracle on the same seeded inputs, and compare."""

from __future__ import annotations

import math

import numpy as np

from long_context_mean_b200 import inputs as I
from oracle import attention as A
from oracle import layout as Y
from oracle import predict as Pr

# Tolerances: attention output max-abs 1e-2 / mean-abs 1e-3 and LSE 1e-3 on
# the same bf16-rounded inputs.  The output is stored in bf16 and the kernel
# multiplies bf16 probabilities, each a relative rounding of 2^-9, so an
# element whose exact value exceeds 1 in magnitude is held to 1e-2 relative
# (max-abs 1e-2 on unit-scale values; a bf16 half-ulp alone is 0.0078 at
# |x| in [2, 4)).  TopCdf decisions exempt within 1e-4 of tau;
# similarity decisions exempt within 1e-5 of theta (fp32 accumulation of a
# 128 x 128 block keeps the mean cosine within ~1e-6); PV-skip decisions
# exempt within 1e-3 of lambda.
OUT_MAX_ABS = 1e-2
OUT_MEAN_ABS = 1e-3
LSE_ABS = 1e-3
TAU_BAND = 1e-4
THETA_BAND = 1e-5
LAMBDA_BAND = 1e-3


def torch_dev():
    import torch
    return torch.device("cuda:0")


def to_dev(x, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(device=torch_dev(), dtype=dtype)


def bf16_dev(bits):
    """bf16 device tensor holding exactly the given bf16 bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(torch_dev())
    return t.view(torch.bfloat16)


def qkv_dev(g, dtype_name):
    import torch
    if dtype_name == "bf16":
        return bf16_dev(g["q_bits"]), bf16_dev(g["k_bits"]), bf16_dev(g["v_bits"])
    return (to_dev(g["q"], torch.float32), to_dev(g["k"], torch.float32), to_dev(g["v"], torch.float32))


def mask_exemptions(orc, sq_dev=None, sk_dev=None, tau=None, theta=0.0, group=1):
    """Blocks where several answers are correct: TopCdf entries within
    TAU_BAND of tau; rows/columns of blocks whose similarity is within
    THETA_BAND of theta."""
    ex = np.zeros(orc["mask"].shape, dtype=bool)
    c = orc["c_excl"]
    with np.errstate(invalid="ignore"):
        ex |= np.abs(c - tau) <= TAU_BAND
    if theta > 0:
        rows = np.abs(orc["s_q"] - theta) <= THETA_BAND            # [B, Hq, nqb]
        cols = np.abs(orc["s_k"] - theta) <= THETA_BAND            # [B, Hkv, nkb]
        cols_q = np.repeat(cols, group, axis=1)
        ex |= rows[..., :, None]
        ex |= cols_q[..., None, :]
        # A key block near theta also changes eligibility -> whole row's TopCdf.
        ex |= cols_q.any(axis=-1)[..., None, None] & np.ones_like(ex)
    return ex


def compare_masks(gpu_mask, orc, tau, theta, group):
    """Exact agreement outside the exemptions; returns the count of
    differing (exempt) blocks."""
    ex = mask_exemptions(orc, tau=tau, theta=theta, group=group)
    diff = gpu_mask != orc["mask"]
    bad = diff & ~ex
    assert not bad.any(), f"{int(bad.sum())} mask blocks differ outside the boundary bands, first at {np.argwhere(bad)[:5]}"
    return int(diff.sum())


def report(label, **fields):
    """Record one parity figure: printed, and appended as a JSON line to the
    file named by SA_PARITY_REPORT when that is set."""
    import json
    import os
    rec = {"case": label, **fields}
    print("parity", json.dumps(rec))
    path = os.environ.get("SA_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def attention_check(out_gpu, lse_gpu, ref, rows=None, label=None):
    """Element-wise comparison on the rows the oracle computed.  The plain
    max-abs is reported beside the held figure (relative above |O| = 1)."""
    o = np.asarray(out_gpu, dtype=np.float64)
    r = ref["out"]
    sel = ~np.isnan(r[..., 0])
    if rows is not None:
        sel &= rows
    d = np.abs(o[sel] - r[sel])
    scaled = d / np.maximum(1.0, np.abs(r[sel]))
    dl = None
    if lse_gpu is not None:
        dl = np.abs(np.asarray(lse_gpu, dtype=np.float64)[sel] - ref["lse"][sel])
    if label is not None:
        report(label, rows=int(sel.sum()), out_max_abs=float(d.max()), out_max_rel_above_1=float(scaled.max()),
               out_mean_abs=float(d.mean()), lse_max_abs=None if dl is None else float(dl.max()))
    assert scaled.max() <= OUT_MAX_ABS, f"max abs (relative above 1) {scaled.max()} (plain max abs {d.max()})"
    assert d.mean() <= OUT_MEAN_ABS, f"mean abs {d.mean()}"
    if dl is not None:
        assert dl.max() <= LSE_ABS, f"lse max abs {dl.max()}"
    return float(d.max()), float(d.mean())


def alpha_report(label, lse_sparse, lse_dense, sel=None):
    """Per-row dropped probability mass alpha = 1 - exp(LSE_sparse -
    LSE_dense) ([P1] 3.2: z = exp(LSE_kept - LSE_full) is the kept mass),
    computed by the oracle; reports mean, max and the worst (b, h, row).
    A restricted softmax keeps at most the full mass, so alpha >= 0 up to the
    two LSEs' tolerance."""
    a = A.dropped_mass_from_lse(lse_sparse, lse_dense)
    if sel is None:
        sel = np.isfinite(a)
    vals = a[sel]
    worst = np.unravel_index(int(np.argmax(np.where(sel, a, -np.inf))), a.shape)
    report(label, alpha_rows=int(sel.sum()), alpha_mean=float(vals.mean()), alpha_max=float(vals.max()),
           alpha_min=float(vals.min()), alpha_worst=[int(x) for x in worst])
    assert vals.min() >= -2 * LSE_ABS, f"alpha {vals.min()} below 0 beyond the LSE tolerance"
    return a


def skip_override_from_gpu(skip_log, row_ptr, col_idx, nqb, B, Hq):
    """Map the GPU's per-tile PV-skip bytes to (b, h, qb, kb) -> bool."""
    out = {}
    for u in range(B * Hq * nqb):
        bh, qb = divmod(u, nqb)
        b, h = divmod(bh, Hq)
        for t in range(row_ptr[u], row_ptr[u + 1]):
            out[(b, h, qb, int(col_idx[t]))] = bool(skip_log[t])
    return out


def check_skip_decisions(gpu_over, orc_skips, orc_gaps, lam):
    """Decisions must agree except within LAMBDA_BAND of lambda."""
    n_band = 0
    for key, s in orc_skips.items():
        if key not in gpu_over:
            continue
        if gpu_over[key] != s:
            assert abs(orc_gaps[key] - lam) <= LAMBDA_BAND, f"skip decision differs off the band at {key}"
            n_band += 1
    return n_band
