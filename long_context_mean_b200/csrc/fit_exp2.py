"""Fits the cubic that the attention kernel uses for part of its exp2 calls.

2^x = 2^n * 2^f with n = round(x) (Cody and Waite's range reduction: the
integer part goes into the exponent field, 2^f is approximated on
[-1/2, 1/2]).  The cubic p(f) = c0 + c1 f + c2 f^2 + c3 f^3 is fitted here to
minimise the largest relative error |p(f) / 2^f - 1| on [-1/2, 1/2]: an
iteratively re-weighted least-squares fit on a dense grid (Lawson's method),
which converges to the minimax (equioscillating) solution.

Run ``python -m long_context_mean_b200.csrc.fit_exp2`` to print the
coefficients (float32-rounded) and the error of the float32 evaluation;
tests/test_exp2_poly.py checks that the kernel source carries these values
and that the float32 emulation of the kernel's bit manipulation stays within
the bound.
"""

from __future__ import annotations

import numpy as np


def fit(degree: int = 3, iters: int = 400):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    w = np.ones_like(f)
    A = np.vander(f, degree + 1, increasing=True)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w) / y
        c, *_ = np.linalg.lstsq(A * sw[:, None], y * sw, rcond=None)
        err = np.abs(A @ c / y - 1.0)
        w = w * (err + 1e-18)
        w /= w.sum()
    return c.astype(np.float32)


def emulate(x, c):
    """float32 evaluation exactly as the kernel does it."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)               # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    n_f = (t - magic).astype(np.float32)
    fr = (x - n_f).astype(np.float32)
    p = np.float32(c[3])
    p = (p * fr + np.float32(c[2])).astype(np.float32)
    p = (p * fr + np.float32(c[1])).astype(np.float32)
    p = (p * fr + np.float32(c[0])).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def max_rel_error(c, lo=-126.0, hi=8.0, n=2000001):
    x = np.linspace(lo, hi, n).astype(np.float32)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(emulate(x, c).astype(np.float64) / ref - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients:", ", ".join(f"{v:.9e}f" for v in c))
    print("max relative error (float32 evaluation on [-126, 8]):", max_rel_error(c))
