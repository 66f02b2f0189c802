"""Pins of the fp64 attention oracle against what the pages and the
mathematics fix (CPU only)."""

import json
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

from oracle import attention as A
from oracle import ledger as L
from long_context_mean_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# The worked example of the error-and-layout page (section 4)
# --------------------------------------------------------------------------

def test_worked_example_reproduces_printed_values():
    g = _gold("worked_example.json")
    ex = inputs.worked_example_inputs()
    m = L.video_masks(4, 4, 4)
    for name, n in g["pairs"].items():
        assert int(m[name].sum()) == n
    assert m["union"].mean() == pytest.approx(g["union_density"], abs=0)
    q, k, v = ex["q"], ex["k"], ex["v"]
    mses = []
    for head in range(2):
        y_full, _, _ = A.masked_attention(q[head], k[head], v, m["full"])
        y_u, _, _ = A.masked_attention(q[head], k[head], v, m["union"])
        mses.append(float(np.mean((y_u - y_full) ** 2)))
    # The page prints the two MSEs to 11 significant digits (5.5294485880e-08,
    # 5.0711107889e-06): the oracle's values, rounded to those digits, are
    # the printed ones (agreement within half a unit of the last digit,
    # about 1e-11 relative).
    for got, printed in zip(mses, g["union_mse"]):
        assert float(f"{got:.10e}") == printed
        assert abs(got - printed) <= 0.5e-10 * 10.0 ** math.floor(math.log10(printed))
    dec = A.error_decomposition(q[0], k[0], v, m["spatial"])
    err = np.linalg.norm(dec["y_tilde"] - dec["y"], axis=-1)
    # printed to 10 decimals (0.0008639397, 0.0117092274)
    assert round(float(err.max()), 10) == g["spatial_head_spatial_mask_max_row_error"]
    assert round(float(dec["bound"].max()), 10) == g["spatial_head_spatial_mask_max_bound"]
    assert np.all(err <= dec["bound"] + 1e-12)


def test_worked_example_permutation_round_trip():
    """Grouping tokens by position (stable argsort by pixel) and undoing it
    returns the same output to fp64 rounding ([P1] section 4)."""
    g = _gold("worked_example.json")
    ex = inputs.worked_example_inputs()
    m = L.video_masks(4, 4, 4)
    perm = np.argsort(ex["pixel"], kind="stable")
    q, k, v = ex["q"][1], ex["k"][1], ex["v"]
    y0, _, _ = A.masked_attention(q, k, v, m["temporal"])
    y1, _, _ = A.masked_attention(q[perm], k[perm], v[perm], m["temporal"][np.ix_(perm, perm)])
    back = np.empty_like(y1)
    back[perm] = y1
    assert np.max(np.abs(back - y0)) <= 4 * g["permutation_max_error"]


def test_counterexample_two_keys():
    g = _gold("worked_example.json")["counterexample"]
    c = inputs.two_key_inputs()
    y, p, _ = A.masked_attention(c["q"], c["k"], c["v"], np.array([[True, True]]))
    yp, _, _ = A.masked_attention(c["q"], c["k"], c["v"], np.array([[True, False]]))
    assert p[0, 0] == pytest.approx(g["retained_mass"], abs=1e-12)
    assert y[0, 0] == pytest.approx(g["dense_output"], abs=1e-12)
    assert yp[0, 0] == pytest.approx(g["pruned_output"], abs=1e-12)
    dec = A.error_decomposition(c["q"], c["k"], c["v"], np.array([[True, False]]))
    assert dec["alpha"][0] == pytest.approx(0.01, abs=1e-12)


def test_empty_row_rejected():
    ex = inputs.worked_example_inputs()
    with pytest.raises(ValueError):
        A.masked_attention(ex["q"][0], ex["k"][0], ex["v"], np.zeros((64, 64), dtype=bool))


# --------------------------------------------------------------------------
# Closed forms and library special cases
# --------------------------------------------------------------------------

def test_all_ones_mask_is_library_softmax():
    rng = np.random.default_rng(1)
    q, k, v = rng.normal(size=(9, 5)), rng.normal(size=(13, 5)), rng.normal(size=(13, 3))
    y, w, lse = A.masked_attention(q, k, v, np.ones((9, 13), dtype=bool))
    s = q @ k.T / math.sqrt(5)
    assert np.allclose(w, softmax(s, axis=1), atol=1e-15)
    assert np.allclose(y, softmax(s, axis=1) @ v, atol=1e-13)
    assert np.allclose(lse, logsumexp(s, axis=1), atol=1e-13)


def test_restricted_softmax_is_renormalised_full_softmax():
    """p_tilde = p / z on the kept set ([P1] section 3.1), checked against
    scipy's softmax of the full row."""
    rng = np.random.default_rng(2)
    q, k, v = rng.normal(size=(7, 4)), rng.normal(size=(11, 4)), rng.normal(size=(11, 2))
    mask = rng.random((7, 11)) < 0.5
    mask[:, 0] = True
    _, w, _ = A.masked_attention(q, k, v, mask)
    p = softmax(q @ k.T / 2.0, axis=1)
    z = (p * mask).sum(axis=1, keepdims=True)
    assert np.allclose(w, np.where(mask, p / z, 0.0), atol=1e-15)


def test_error_identity_and_bound_random():
    rng = np.random.default_rng(3)
    for _ in range(20):
        n, d, dv = rng.integers(3, 20), rng.integers(1, 8), rng.integers(1, 4)
        q, k, v = rng.normal(size=(n, d)) * 2, rng.normal(size=(n, d)) * 2, rng.normal(size=(n, dv)) * 5
        mask = rng.random((n, n)) < 0.4
        mask[np.arange(n), rng.integers(0, n, n)] = True
        dec = A.error_decomposition(q, k, v, mask)
        diff = dec["y_tilde"] - dec["y"]
        some = dec["alpha"] > 1e-14
        assert np.allclose(diff[some], (dec["alpha"][:, None] * (dec["r"] - dec["u"]))[some], atol=1e-12)
        assert np.all(np.linalg.norm(diff, axis=1) <= dec["bound"] + 1e-12)


def test_error_identity_hand_expanded_three_keys():
    """Brute force on one row with three keys, written out term by term."""
    s = np.array([0.3, -1.2, 2.0])
    v = np.array([[1.0], [-4.0], [2.5]])
    e = np.exp(s)
    p = e / e.sum()
    keep = np.array([True, False, True])
    y = p @ v
    yt = (e[0] * v[0] + e[2] * v[2]) / (e[0] + e[2])
    alpha = p[1]
    dec = A.error_decomposition(s[None, :1] * 0 + 1.0, s[:, None], v, keep[None, :], scale=1.0)
    assert dec["y"][0] == pytest.approx(y, abs=1e-14)
    assert dec["y_tilde"][0] == pytest.approx(yt, abs=1e-14)
    assert dec["alpha"][0] == pytest.approx(alpha, abs=1e-15)
    assert (yt - y)[0] == pytest.approx(alpha * (yt[0] - v[1, 0]), abs=1e-13)


# --------------------------------------------------------------------------
# Tile recurrence vs one-shot definitions
# --------------------------------------------------------------------------

def _random_block_mask(rng, nqb, nkb, p=0.4, causal=False, n=None, bq=None, bk=None):
    m = rng.random((nqb, nkb)) < p
    for qb in range(nqb):
        if causal:
            last = min(n, (qb + 1) * bq) - 1
            valid = np.arange(nkb) * bk <= last
            m[qb] &= valid
            m[qb, 0] = True          # key 0 is visible to every row
        elif not m[qb].any():
            m[qb, rng.integers(nkb)] = True
    return m


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,bq,bk", [(37, 8, 4), (64, 16, 16), (50, 16, 8)])
def test_block_sparse_lambda_off_is_restricted_softmax(causal, n, bq, bk):
    rng = np.random.default_rng(n * 7 + causal)
    d, dv = 6, 5
    q, k, v = rng.normal(size=(n, d)), rng.normal(size=(n, d)), rng.normal(size=(n, dv))
    nqb, nkb = -(-n // bq), -(-n // bk)
    kept = _random_block_mask(rng, nqb, nkb, causal=causal, n=n, bq=bq, bk=bk)
    r = A.block_sparse_attention(q, k, v, kept, bq, bk, causal=causal)
    tok = A.kept_blocks_to_token_mask(kept, n, bq, bk, causal)
    y, _, lse = A.masked_attention(q, k, v, tok)
    assert np.allclose(r["out"], y, atol=1e-13)
    assert np.allclose(r["lse"], lse, atol=1e-13)
    assert not any(r["skips"].values())


def test_all_kept_equals_dense_causal():
    rng = np.random.default_rng(11)
    n, bq, bk = 45, 16, 8
    q, k, v = rng.normal(size=(n, 4)), rng.normal(size=(n, 4)), rng.normal(size=(n, 3))
    nqb, nkb = -(-n // bq), -(-n // bk)
    kept = np.array([[kb * bk <= min(n, (qb + 1) * bq) - 1 for kb in range(nkb)] for qb in range(nqb)])
    r = A.block_sparse_attention(q, k, v, kept, bq, bk, causal=True)
    s = q @ k.T / 2.0
    s[np.triu_indices(n, 1)] = -np.inf
    assert np.allclose(r["out"], softmax(s, axis=1) @ v, atol=1e-13)
    assert np.allclose(r["lse"], logsumexp(s, axis=1), atol=1e-13)


def _brute_pv_skip(q, k, v, kept, bq, bk, lam, causal):
    """Restatement without the recurrence: the running maximum before tile t
    is the max over the earlier kept tiles; a tile is skipped when the
    largest (tile max - running max) over the q-block's rows is < lam; the
    output drops the skipped tiles from the numerator only."""
    n, d = q.shape
    s_all = q @ k.T / math.sqrt(d)
    if causal:
        s_all[np.triu_indices(n, 1)] = -np.inf
    out = np.zeros((n, v.shape[1]))
    skips = {}
    for qb in range(kept.shape[0]):
        i0, i1 = qb * bq, min(n, (qb + 1) * bq)
        cols = np.flatnonzero(kept[qb])
        tiles = [(kb, kb * bk, min(n, (kb + 1) * bk)) for kb in cols]
        skipped = []
        for t, (kb, j0, j1) in enumerate(tiles):
            gaps = []
            for i in range(i0, i1):
                cur = s_all[i, j0:j1].max()
                if not np.isfinite(cur):
                    continue
                prev = max([s_all[i, a:b].max() for (_, a, b) in tiles[:t]], default=-np.inf)
                gaps.append(cur - max(prev, cur))
            gap = max(gaps) if gaps else -np.inf
            skips[(qb, int(kb))] = gap < lam
            if gap < lam:
                skipped.append(kb)
        for i in range(i0, i1):
            num = np.zeros(v.shape[1])
            den = 0.0
            mf = max(s_all[i, a:b].max() for (_, a, b) in tiles)
            for kb, a, b in tiles:
                w = np.exp(s_all[i, a:b] - mf)
                den += w.sum()
                if kb not in skipped:
                    num += w @ v[a:b]
            out[i] = num / den
    return out, skips


@pytest.mark.parametrize("lam,causal", [(-1.0, False), (-3.0, True), (0.0, False), (-0.5, True)])
def test_pv_skip_matches_brute_force(lam, causal):
    rng = np.random.default_rng(int(abs(lam) * 10) + causal)
    n, bq, bk, d = 48, 16, 8, 4
    # Every query leans on one direction u and the keys' weight on u falls
    # along the sequence, so later tiles sit well below the running max.
    u = np.ones(d)
    q = 2.0 * u + 0.3 * rng.normal(size=(n, d))
    k = np.linspace(3, -3, n)[:, None] * u + 0.3 * rng.normal(size=(n, d))
    v = rng.normal(size=(n, 3))
    nqb, nkb = n // bq, n // bk
    kept = _random_block_mask(rng, nqb, nkb, p=0.7, causal=causal, n=n, bq=bq, bk=bk)
    r = A.block_sparse_attention(q, k, v, kept, bq, bk, causal=causal, lam=lam)
    ref, skips = _brute_pv_skip(q, k, v, kept, bq, bk, lam, causal)
    assert r["skips"] == skips
    assert np.allclose(r["out"], ref, atol=1e-12)
    if lam < 0:
        assert any(skips.values()), "case should exercise the skip"


def test_override_only_on_the_band():
    rng = np.random.default_rng(5)
    n, bq, bk = 32, 16, 8
    q, k, v = rng.normal(size=(n, 4)), rng.normal(size=(n, 4)), rng.normal(size=(n, 2))
    kept = np.ones((2, 4), dtype=bool)
    r = A.block_sparse_attention(q, k, v, kept, bq, bk, lam=-2.0)
    key, gap = next(iter(r["gaps"].items()))
    with pytest.raises(ValueError):
        A.block_sparse_attention(q, k, v, kept, bq, bk, lam=-2.0,
                                 skip_override={key: not r["skips"][key]})
    # Put lambda exactly on that tile's gap: flipping it is then allowed.
    r2 = A.block_sparse_attention(q, k, v, kept, bq, bk, lam=gap,
                                  skip_override={key: True})
    assert r2["skips"][key] is True


def test_dropped_mass_from_lse():
    ex = inputs.worked_example_inputs()
    m = L.video_masks(4, 4, 4)
    _, _, lse_full = A.masked_attention(ex["q"][0], ex["k"][0], ex["v"], m["full"])
    _, _, lse_s = A.masked_attention(ex["q"][0], ex["k"][0], ex["v"], m["temporal"])
    dec = A.error_decomposition(ex["q"][0], ex["k"][0], ex["v"], m["temporal"])
    assert np.allclose(A.dropped_mass_from_lse(lse_s, lse_full), dec["alpha"], atol=1e-12)
