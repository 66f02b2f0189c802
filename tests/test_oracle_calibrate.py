"""Pins of the oracle's per-layer calibration ([P3] section 2.4): the
relative L1 definition on closed-form arrays, the selection rule on
hand-made tables, and the search on a small problem (the full-mask point
reproduces dense attention; the chosen point is feasible and as sparse as
any feasible point)."""

import math

import numpy as np
import pytest

from long_context_mean_b200 import inputs as I
from oracle import calibrate as C


def test_relative_l1_closed_form():
    assert C.relative_l1([1.0, -2.0, 3.0], [1.0, -1.0, 1.0]) == pytest.approx(3.0 / 6.0, abs=1e-15)
    assert C.relative_l1([[2.0, 0.0]], [[2.0, 0.0]]) == 0.0
    assert C.relative_l1([0.0, 0.0], [1.0, 1.0]) == 0.0   # no reference mass: defined as 0


def test_select_tau_theta_table():
    rows = [
        {"tau": 1.0, "theta": 0.0, "l1": 0.0, "sparsity": 0.0},
        {"tau": 0.9, "theta": 0.0, "l1": 0.02, "sparsity": 0.5},
        {"tau": 0.5, "theta": 0.0, "l1": 0.049, "sparsity": 0.7},
        {"tau": 0.3, "theta": 0.0, "l1": 0.06, "sparsity": 0.9},     # infeasible at 0.05
        {"tau": 0.5, "theta": 0.4, "l1": 0.04, "sparsity": 0.7},     # same sparsity, smaller error
        {"tau": 0.6, "theta": 0.4, "l1": 0.04, "sparsity": 0.7},     # tie on error: larger tau wins
    ]
    best = C.select_tau_theta(rows, 0.05)
    assert (best["tau"], best["theta"]) == (0.6, 0.4)
    assert C.select_tau_theta(rows, 0.0) is None                       # strict bound
    assert C.select_tau_theta(rows, 0.001)["tau"] == 1.0


def test_select_lambda_table():
    rows = [
        {"lam": -math.inf, "l1": 0.03, "pv_skip": 0.0},
        {"lam": -8.0, "l1": 0.031, "pv_skip": 0.1},
        {"lam": -4.0, "l1": 0.05, "pv_skip": 0.3},
        {"lam": -2.0, "l1": 0.07, "pv_skip": 0.5},
    ]
    assert C.select_lambda(rows, 0.06)["lam"] == -4.0
    assert C.select_lambda(rows, 0.031)["lam"] == -math.inf
    rows.append({"lam": -5.0, "l1": 0.05, "pv_skip": 0.3})                # tie: larger lambda wins
    assert C.select_lambda(rows, 0.06)["lam"] == -4.0


def small_problem():
    w = I.Workload("calib_small", 91, 1, 2, 2, 1, 1, 384, 0, 16, 16, "fp32", "field", bq=64, bk=64,
                   sigma=(0.0, 0.0, 10.0), sigma_pos=30.0)
    g = I.gen_qkv(w)
    return w, g


def test_calibration_search_small():
    w, g = small_problem()
    taus, thetas = [0.3, 0.6, 0.9, 1.0], [0.0, 0.3]
    lams = [-math.inf, -8.0, -4.0, -2.0, -1.0]
    res = C.calibrate(g["q"], g["k"], g["v"], w.bq, w.bk, taus, thetas, lams, l1=0.05, l2=0.06)
    full = [r for r in res["step1"] if r["tau"] == 1.0 and r["theta"] == 0.0][0]
    assert full["sparsity"] == 0.0 and full["l1"] < 1e-12          # every block kept = dense attention
    feas = [r for r in res["step1"] if r["l1"] < 0.05]
    chosen = [r for r in res["step1"] if (r["tau"], r["theta"]) == (res["tau"], res["theta"])][0]
    assert chosen["l1"] < 0.05
    assert all(chosen["sparsity"] >= r["sparsity"] for r in feas)
    lam_row = [r for r in res["step2"] if r["lam"] == res["lam"]][0]
    assert lam_row["l1"] < 0.06
    inf_row = [r for r in res["step2"] if r["lam"] == -math.inf][0]
    assert inf_row["pv_skip"] == 0.0 and inf_row["l1"] == pytest.approx(chosen["l1"], abs=1e-14)
    assert all(lam_row["pv_skip"] >= r["pv_skip"] for r in res["step2"] if r["l1"] < 0.06)
