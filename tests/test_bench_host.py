"""Host-side arithmetic of bench.py on CPU: the kept-block FLOP count that
the headline metric divides by the step time, checked against brute-force
pair counting, and the workload description of the JSON line."""

import types

import numpy as np
import pytest

import bench
from long_context_mean_b200 import inputs as I


def _random_csr(rng, R, nkb, p):
    rows = [np.flatnonzero(rng.random(nkb) < p) for _ in range(R)]
    rows = [r if r.size else np.array([0]) for r in rows]
    row_ptr = np.concatenate([[0], np.cumsum([r.size for r in rows])]).astype(np.int64)
    col_idx = np.concatenate(rows).astype(np.int32)
    return row_ptr, col_idx


def _brute(w, row_ptr, col_idx, skip, nqb):
    qk = pv = 0
    for u in range(len(row_ptr) - 1):
        qb = u % nqb
        for t in range(row_ptr[u], row_ptr[u + 1]):
            kb = int(col_idx[t])
            pairs = 0
            for i in range(qb * w.bq, min(w.N, (qb + 1) * w.bq)):
                for j in range(kb * w.bk, min(w.N, (kb + 1) * w.bk)):
                    if not w.causal or j <= i:
                        pairs += 1
            qk += 2 * w.d * pairs
            if not skip[t]:
                pv += 2 * w.dv * pairs
    return float(qk), float(pv)


@pytest.mark.parametrize("causal", [False, True])
def test_kept_flops_is_the_pair_count(causal):
    rng = np.random.default_rng(3 + causal)
    w = types.SimpleNamespace(N=300, bq=128, bk=64, d=128, dv=96, causal=causal)
    nqb, nkb = 3, 5
    row_ptr, col_idx = _random_csr(rng, 2 * nqb, nkb, 0.6)
    skip = (rng.random(col_idx.size) < 0.3).astype(np.uint8)
    got = bench.kept_flops(w, row_ptr, col_idx, skip, nqb)
    assert got == pytest.approx(_brute(w, row_ptr, col_idx, skip, nqb), rel=0, abs=0)


def test_workload_config_names_the_sizes():
    w = I.WORKLOADS["video"]
    c = bench.workload_config(w, 2)
    assert c["seq_len"] == w.N == 20506 and c["global_batch"] == 2 * w.B
    assert "N=20506" in c["workload"] and "[13,30,52]+226" in c["workload"]
    assert c["parallelism"] == "replicas x2" and "flushed" in c["l2"]


def test_cpu_baseline_samples_heads_in_turn():
    """The CPU baseline walks query heads in turn and reads each one's own kv
    head (GQA), timing only the oracle's attention."""
    w = I.WORKLOADS["toy"].with_(Hq=4, Hkv=2, generator="lowrank", rank=4, sigma_pos=4.0)
    g = I.gen_qkv(w)
    q, k, v, m = bench.oracle_sample_setup(w, g, head=3)
    from oracle import layout as Y
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    assert np.array_equal(q, Y.reorder(g["q"][:1, 3:4], perm))
    assert np.array_equal(k, Y.reorder(g["k"][:1, 1:2], perm))
    assert np.array_equal(v, Y.reorder(g["v"][:1, 1:2], perm))
    r = bench.cpu_baseline(w, g, seconds=1e9)     # every block of every head
    nqb = -(-w.N // w.bq)
    assert f"of {4 * nqb} random query blocks of query heads 0-3" in r["sample"]
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1
