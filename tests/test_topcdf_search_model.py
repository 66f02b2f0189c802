"""A float32 model of the TopCdf threshold search that score_topcdf_kernel
runs on rows it cannot settle by its arg-max loop, checked on the CPU against
the oracle's sorted rule ([P3] SpargeAttention notes, 2.2: keep an entry while
the mass sorted before it is below tau times the row's total).

The kernel never sorts a row.  It looks for t*, the smallest fp32 bit pattern
whose mass of larger probabilities, f(t), is below tau * total:

1. one pass sums the row and counts the p above a lower start
   e = (1 - tau) / (4 n) (0 when 1 - tau < 1e-3);
2. bisection over the bit patterns while more than 128 p lie between the
   bounds;
3. the remaining candidates are gathered (four per lane, in block order) and
   each further step tests one candidate strictly inside the bounds, taken
   from a rotating lane, with f = f(hi on entry) + the candidates' mass
   above t.

Blocks above t* are kept, and blocks equal to t* in index order while
f(t*) + rank * t* < tau * total.  The model repeats these steps in numpy
float32.  Its sums run in another order than the warp's, which can move a
decision only where f(t) meets the limit within rounding, well inside the
1e-4 band of cumulative mass that the GPU tests exempt.  The tests check the
reasoning behind the steps: the start e clears the limit, both finishes
reach the same boundary, and the kept set is the sorted rule's, on rows with
ties, a single value, one dominant entry, a boundary inside a flat tail just
above the start, and tau at its edges.
"""

import numpy as np
import pytest

from oracle import predict as Pr

NCAND = 128      # candidates the kernel gathers into registers (4 per lane)
TAU_BAND = 1e-4  # the GPU tests' exemption band of cumulative mass


def _bits(p):
    return np.asarray(p, dtype=np.float32).view(np.uint32)


def _f32sum(x):
    return np.float32(np.sum(np.asarray(x, dtype=np.float32), dtype=np.float32))


def lower_start(tau, n):
    """The kernel's first bisection bound (as a bit pattern)."""
    if np.float32(tau) > np.float32(0.999):
        return 0
    e = np.float32(0.25) * (np.float32(1.0) - np.float32(tau)) / np.float32(n)
    return int(_bits(e))


def kernel_search(p, tau, finish="candidates"):
    """The kernel's kept set for one row of probabilities p in [0, 1] whose
    largest entry is 1.  finish="candidates" is the kernel's last phase;
    finish="bisect" continues the bisection there instead (the earlier form),
    for comparing the two."""
    p = np.asarray(p, dtype=np.float32)
    b = _bits(p)
    n4 = -(-p.size // 4) * 4                      # the kernel pads rows to 4
    lo = lower_start(tau, n4)
    total = _f32sum(p[b > 0])
    limit = np.float32(tau) * total
    c_lo = int((b > lo).sum())
    hi, f_hi, c_hi = 0x3F800000, np.float32(0.0), 0
    while hi - lo > 1 and c_lo - c_hi > NCAND:
        mid = lo + (hi - lo) // 2
        sel = b > mid
        m, c = _f32sum(p[sel]), int(sel.sum())
        if m < limit:
            hi, f_hi, c_hi = mid, m, c
        else:
            lo, c_lo = mid, c
    if hi - lo > 1:
        cand = p[(b > lo) & (b <= hi)]
        assert cand.size <= NCAND
        cb = _bits(cand)
        f_base = f_hi
        if finish == "bisect":
            while hi - lo > 1:
                mid = lo + (hi - lo) // 2
                m = np.float32(f_base + _f32sum(cand[cb > mid]))
                if m < limit:
                    hi, f_hi = mid, m
                else:
                    lo = mid
        else:
            step = 0
            while True:
                # candidate j sits in lane j % 32, register j // 32; a lane
                # offers its lowest register strictly inside (lo, hi)
                offer = {}
                for j in range(cand.size):
                    if lo < int(cb[j]) < hi and (j % 32) not in offer:
                        offer[j % 32] = int(cb[j])
                if not offer:
                    break
                rot = (step * 13) & 31
                mid = offer[min(offer, key=lambda lane: (lane - rot) % 32)]
                m = np.float32(f_base + _f32sum(cand[cb > mid]))
                if m < limit:
                    hi, f_hi = mid, m
                else:
                    lo = mid
                step += 1
    vstar = np.uint32(hi).view(np.float32)
    keep = b > hi
    run = 0
    for kb in np.flatnonzero(b == hi):
        keep[kb] = np.float32(f_hi + np.float32(run) * vstar) < limit
        run += 1
    return keep


def _row(rng, n, kind, tau=0.5):
    if kind == "spread":
        s = rng.normal(0.0, rng.uniform(0.3, 5.0), n)
    elif kind == "ties":
        s = np.round(rng.normal(0.0, 2.0, n) * 2.0) / 2.0
    elif kind == "flat":
        s = np.zeros(n)
    elif kind == "dominant":
        s = rng.normal(0.0, 0.5, n)
        s[rng.integers(n)] += 30.0
    elif kind == "tail":
        # one entry of 1 and a flat tail holding 2 (1 - tau) / tau of mass
        # (each tail entry at most 1/2): on long rows the boundary falls
        # inside the tail, a few times above the start e
        x = 2.0 * (1.0 - tau) / (tau * max(n - 1, 1)) if tau < 1.0 else 1e-3
        p = np.full(n, min(x, 0.5))
        p[rng.integers(n)] = 1.0
        return p.astype(np.float32)
    else:
        raise ValueError(kind)
    return np.exp(s - s.max()).astype(np.float32)


TAUS = [0.01, 0.25, 0.5, 0.9, 0.95, 0.999, 0.9995, 1.0]


@pytest.mark.parametrize("tau", TAUS)
def test_lower_start_clears_the_limit(tau):
    """f(e) >= tau * total on every row: the p <= e hold at most (1 - tau)/4
    of a total that is at least max p = 1."""
    rng = np.random.default_rng(int(tau * 1e4))
    for n in (1, 3, 64, 777, 2048, 4095):
        for kind in ("spread", "ties", "flat", "dominant", "tail"):
            p = _row(rng, n, kind, tau)
            b = _bits(p)
            n4 = -(-n // 4) * 4
            lo = lower_start(tau, n4)
            limit = np.float32(tau) * _f32sum(p[b > 0])
            assert _f32sum(p[b > lo]) >= limit


@pytest.mark.parametrize("tau", TAUS)
def test_search_keeps_the_sorted_rule_set(tau):
    rng = np.random.default_rng(17 + int(tau * 1e4))
    for trial in range(60):
        n = int(rng.choice([1, 2, 5, 129, 600, 2048, int(rng.integers(1, 4096))]))
        kind = ("spread", "ties", "flat", "dominant", "tail")[trial % 5]
        p = _row(rng, n, kind, tau)
        kept, c = Pr.topcdf(p.astype(np.float64), tau)
        got = kernel_search(p, tau)
        band = np.abs(c - tau) <= TAU_BAND
        bad = (got != kept) & ~band
        assert not bad.any(), (n, kind, np.flatnonzero(bad)[:5])


def test_candidate_steps_reach_the_bisection_boundary():
    """The last phase's two forms give the same set (f only changes at a
    candidate's value, so both stop at the same t*)."""
    rng = np.random.default_rng(5)
    for trial in range(120):
        n = int(rng.integers(200, 4096))
        p = _row(rng, n, ("spread", "ties", "dominant")[trial % 3])
        tau = float(rng.choice([0.25, 0.5, 0.9, 0.95, 0.9995]))
        assert np.array_equal(kernel_search(p, tau), kernel_search(p, tau, finish="bisect"))


def test_worked_row():
    """The notes' small example: [0.6, 0.3, 0.1] at tau = 0.8 keeps the
    first two (their sorted exclusive masses 0 and 0.6 are below 0.8)."""
    p = np.array([0.6, 0.3, 0.1], dtype=np.float32) / np.float32(0.6)
    assert kernel_search(p, 0.8).tolist() == [True, True, False]
