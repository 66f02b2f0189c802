"""GPU parity of the per-head spatial / temporal path (sa_head_placement,
sa_reorder_heads, sa_rows_mse, block-sparse attention with one output
permutation per head, and the online profile) against oracle.svg."""

import numpy as np
import pytest

from long_context_mean_b200 import inputs as I
from oracle import attention as A
from oracle import svg as S
from tests import _parity as P

pytestmark = pytest.mark.gpu

SMALL = dict(T=4, Hg=8, Wg=12, txt=37)        # nv = 384, N = 421: 4 query tiles, a ragged tail


def _placement(T, Hg, Wg, txt, kinds, bq, bk):
    import torch
    from long_context_mean_b200 import sa
    n = T * Hg * Wg + txt
    nqb, nkb = -(-n // bq), -(-n // bk)
    kd = torch.tensor(kinds, dtype=torch.int32, device="cuda")
    perms = torch.empty(len(kinds), n, dtype=torch.int32, device="cuda")
    bm = torch.empty(len(kinds), nqb, nkb, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.head_placement(T, Hg, Wg, txt, kd, bq, bk, perms, bm, st)
    return perms.cpu().numpy(), bm.cpu().numpy().astype(bool), sa.read_status(st)


@pytest.mark.parametrize("T,Hg,Wg,txt,bq,bk", [(3, 4, 5, 7, 8, 4), (4, 8, 12, 37, 128, 64),
                                               (13, 6, 7, 20, 128, 128), (2, 1, 1, 0, 1, 1)])
def test_head_placement_is_the_oracle(T, Hg, Wg, txt, bq, bk):
    kinds = [S.SPATIAL, S.TEMPORAL, S.TEMPORAL, S.SPATIAL]
    perms, bm, st = _placement(T, Hg, Wg, txt, kinds, bq, bk)
    assert st == 0
    for h, c in enumerate(kinds):
        assert np.array_equal(perms[h], S.candidate_order(T, Hg, Wg, txt, c))
        assert np.array_equal(bm[h], S.head_block_mask(T, Hg, Wg, txt, c, bq, bk))


def test_head_placement_rejects_unknown_kind():
    perms, bm, st = _placement(2, 2, 2, 1, [S.SPATIAL, 7], 4, 4)
    from long_context_mean_b200 import sa
    assert st == sa.SA_ERR_INVALID_ARG
    assert not bm[1].any() and bm[0].any()
    assert np.array_equal(perms[1], np.arange(9))


def test_reorder_heads_gathers_per_head():
    import torch
    from long_context_mean_b200 import sa
    T, Hg, Wg, txt = 3, 4, 5, 7
    kinds = [S.TEMPORAL, S.SPATIAL, S.TEMPORAL]
    perms, _, _ = _placement(T, Hg, Wg, txt, kinds, 8, 8)
    n = perms.shape[1]
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 3, n, 40)).astype(np.float32)
    bits = I.to_bf16_bits(x)
    xd = P.bf16_dev(bits)
    y = torch.empty_like(xd)
    sa.reorder_heads(torch.from_numpy(perms).cuda(), xd, y)
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    for h in range(3):
        assert np.array_equal(got[0, h], bits[0, h][perms[h]])


def test_rows_mse_is_the_oracle():
    import torch
    from long_context_mean_b200 import sa
    rng = np.random.default_rng(9)
    BH, n, dv = 5, 300, 72
    a = I.to_bf16_bits(rng.standard_normal((BH, n, dv)).astype(np.float32))
    b = I.to_bf16_bits(rng.standard_normal((BH, n, dv)).astype(np.float32))
    rows = rng.integers(0, n, size=33)
    rows[1] = rows[0]                                    # a repeated row counts twice
    out = torch.zeros(BH, dtype=torch.float64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.rows_mse(P.bf16_dev(a), P.bf16_dev(b), torch.from_numpy(rows.astype(np.int32)).cuda(), out, st)
    assert sa.read_status(st) == 0
    af, bf = I.bf16_bits_to_f32(a), I.bf16_bits_to_f32(b)
    for h in range(BH):
        assert float(out[h]) == pytest.approx(S.sampled_mse(af[h], bf[h], rows), rel=1e-12)
    bad = torch.tensor([0, n], dtype=torch.int32, device="cuda")
    sa.rows_mse(P.bf16_dev(a), P.bf16_dev(b), bad, out, st)
    assert sa.read_status(st) == sa.SA_ERR_INVALID_ARG


@pytest.mark.parametrize("dt,d,Hq,Hkv", [("bf16", 128, 4, 2), ("fp32", 64, 2, 2)])
def test_rows_attn_dense_vs_oracle(dt, d, Hq, Hkv):
    """Sampled rows (with a repeat and both ends) against the dense softmax."""
    import torch
    from long_context_mean_b200 import sa
    N = 421
    w = I.Workload("rows", 77, 1, Hq, Hkv, 1, 1, N, 0, d, d, dt, "iid")
    g = I.gen_qkv(w)
    q, k, v = P.qkv_dev(g, dt)
    rows = np.array([0, N - 1, 200, 200, 17, 399], dtype=np.int32)
    out = torch.empty(Hq, rows.size, d, dtype=torch.float32, device="cuda")
    lse = torch.empty(Hq, rows.size, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.rows_attn(q, k, v, sa.make_shape(q, k, v), torch.from_numpy(rows).cuda(), out, lse, status=st)
    assert sa.read_status(st) == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for h in range(Hq):
        y, _, l = A.masked_attention(g["q"][0, h][rows], g["k"][0, h // (Hq // Hkv)], g["v"][0, h // (Hq // Hkv)],
                                     np.ones((rows.size, N), bool))
        assert np.abs(out[h] - y).max() < 1e-4
        assert np.abs(lse[h] - l).max() < 1e-4


def test_rows_attn_candidates_vs_oracle():
    """Sampled rows under each head's candidate (placement from the GPU)
    against the oracle's candidate attention at those rows."""
    import torch
    from long_context_mean_b200 import sa
    T, Hg, Wg, txt = SMALL["T"], SMALL["Hg"], SMALL["Wg"], SMALL["txt"]
    bias = ["frame", "position", "position", "frame"]
    kinds = [S.SPATIAL, S.TEMPORAL, S.SPATIAL, S.TEMPORAL]
    g = I.biased_video_heads(T, Hg, Wg, txt, bias, seed=5)
    q, k, v = (P.bf16_dev(g[n + "_bits"]) for n in "qkv")
    n = T * Hg * Wg + txt
    perms = torch.empty(4, n, dtype=torch.int32, device="cuda")
    bm = torch.empty(4, -(-n // 128), -(-n // 64), dtype=torch.uint8, device="cuda")
    kd = torch.tensor(kinds, dtype=torch.int32, device="cuda")
    sa.head_placement(T, Hg, Wg, txt, kd, 128, 64, perms, bm)
    rows = np.array([0, 5, 130, 383, 384, 420, 250], dtype=np.int32)
    out = torch.empty(4, rows.size, 128, dtype=torch.float32, device="cuda")
    lse = torch.empty(4, rows.size, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.rows_attn(q, k, v, sa.make_shape(q, k, v), torch.from_numpy(rows).cuda(), out, lse, perms, bm, 128, 64,
                 status=st)
    assert sa.read_status(st) == 0
    out_h, lse_h = out.cpu().numpy(), lse.cpu().numpy()
    for h, c in enumerate(kinds):
        y, l = S.candidate_attention(g["q"][0, h], g["k"][0, h], g["v"][0, h], T, Hg, Wg, txt, c, 128, 64)
        assert np.abs(out_h[h] - y[rows]).max() < 1e-4
        assert np.abs(lse_h[h] - l[rows]).max() < 1e-4
    bad = torch.tensor([0, n], dtype=torch.int32, device="cuda")
    out2 = torch.empty(4, 2, 128, dtype=torch.float32, device="cuda")
    sa.rows_attn(q, k, v, sa.make_shape(q, k, v), bad, out2, None, perms, bm, 128, 64, status=st)
    assert sa.read_status(st) == sa.SA_ERR_INVALID_ARG


def _small_pipe(bias, flags=0, **kw):
    from long_context_mean_b200 import svg
    g = I.biased_video_heads(SMALL["T"], SMALL["Hg"], SMALL["Wg"], SMALL["txt"], bias, seed=11)
    pipe = svg.SvgPipeline(1, len(bias), SMALL["T"], SMALL["Hg"], SMALL["Wg"], SMALL["txt"], 128, 128,
                           flags=flags, **kw)
    return g, pipe


@pytest.mark.parametrize("flags", [0, 1])
def test_run_matches_oracle_small(flags):
    bias = ["frame", "position", "position", "frame"]
    kinds = [S.SPATIAL, S.TEMPORAL, S.SPATIAL, S.TEMPORAL]     # two heads on the wrong candidate
    g, pipe = _small_pipe(bias, flags)
    pipe.place(kinds)
    out, lse = pipe.run(P.bf16_dev(g["q_bits"]), P.bf16_dev(g["k_bits"]), P.bf16_dev(g["v_bits"]))
    assert pipe.status() == 0
    ref_out, ref_lse = S.svg_attention(g["q"][0], g["k"][0], g["v"][0], kinds, SMALL["T"], SMALL["Hg"],
                                       SMALL["Wg"], SMALL["txt"], 128, 64)
    P.attention_check(out.float().cpu().numpy()[0], lse.cpu().numpy()[0, ..., 0],
                      {"out": ref_out, "lse": ref_lse})


def test_profile_picks_the_oracle_choice_small():
    bias = ["frame", "position", "frame", "position", "position"]
    g, pipe = _small_pipe(bias, nrows=32, seed=3)
    q, k, v = (P.bf16_dev(g[n + "_bits"]) for n in "qkv")
    choice, mse = pipe.profile(q, k, v)
    rows = pipe.rows.cpu().numpy()
    ref_choice, ref_mse = S.select_heads(g["q"][0], g["k"][0], g["v"][0], SMALL["T"], SMALL["Hg"], SMALL["Wg"],
                                         SMALL["txt"], 128, 64, rows)
    assert choice == ref_choice.tolist() == [S.SPATIAL, S.TEMPORAL, S.SPATIAL, S.TEMPORAL, S.TEMPORAL]
    mse = mse.numpy()
    for h, c in enumerate(choice):
        lose = 1 - c
        # the losing candidate's error is large and computed alike; the
        # winner's sits at the bf16 rounding of the outputs
        assert mse[lose, h] == pytest.approx(ref_mse[lose, h], rel=0.05)
        assert mse[c, h] < 1e-4 and ref_mse[c, h] < 1e-4
    # the placed choice is what run() executes
    out, lse = pipe.run(q, k, v)
    ref_out, ref_lse = S.svg_attention(g["q"][0], g["k"][0], g["v"][0], choice, SMALL["T"], SMALL["Hg"],
                                       SMALL["Wg"], SMALL["txt"], 128, 64)
    P.attention_check(out.float().cpu().numpy()[0], lse.cpu().numpy()[0, ..., 0],
                      {"out": ref_out, "lse": ref_lse})


def _row_reference(q, k, v, i, T, Hg, Wg, txt, kind, bq, bk):
    """fp64 output and lse of original row i under a candidate: the keys of
    the kept tiles of its query block (block cover taken from the oracle's
    element mask rows), through the restricted softmax."""
    perm = S.candidate_order(T, Hg, Wg, txt, kind)
    n = perm.size
    place = int(np.flatnonzero(perm == i)[0])
    qb = place // bq
    rows = perm[qb * bq:(qb + 1) * bq]
    m = S.element_mask_rows(T, Hg, Wg, txt, kind, rows)[:, perm]       # the q-block's rows in the head's order
    nkb = -(-n // bk)
    keep = np.zeros(n, dtype=bool)
    for kb in range(nkb):
        if m[:, kb * bk:(kb + 1) * bk].any():
            keep[kb * bk:(kb + 1) * bk] = True
    mask = np.zeros((1, n), dtype=bool)
    mask[0, perm[keep]] = True
    y, _, lse = A.masked_attention(q[i:i + 1], k, v, mask)
    return y[0], lse[0]


def test_full_size_video_profile_and_sampled_rows():
    """The video shape (13 x 30 x 52 latent, 226 text tokens, 24 heads):
    the profile recovers each head's bias, and sampled rows of the run match
    the restricted softmax over their kept tiles."""
    from long_context_mean_b200 import svg
    w = I.WORKLOADS["video"]
    bias = ["frame" if h % 3 else "position" for h in range(w.Hq)]
    g = I.biased_video_heads(w.T, w.H, w.W, w.txt_len, bias, seed=21)
    pipe = svg.svg_pipeline_for(w)
    q, k, v = (P.bf16_dev(g[n + "_bits"]) for n in "qkv")
    choice, _ = pipe.profile(q, k, v)
    assert choice == [S.SPATIAL if b == "frame" else S.TEMPORAL for b in bias]
    out, lse = pipe.run(q, k, v)
    assert pipe.status() == 0
    out = out.float().cpu().numpy()[0]
    lse = lse.cpu().numpy()[0, ..., 0]
    rng = np.random.default_rng(4)
    n = w.N
    for h in (0, 1, 2, 23):
        qh, kh, vh = (g[x][0, h].astype(np.float64) for x in "qkv")
        for i in list(rng.integers(0, n, size=5)) + [0, n - 1, w.T * w.H * w.W]:
            y, l = _row_reference(qh, kh, vh, int(i), w.T, w.H, w.W, w.txt_len, choice[h], w.bq, w.bk)
            d = np.abs(out[h, i] - y) / np.maximum(1.0, np.abs(y))
            assert d.max() <= P.OUT_MAX_ABS, (h, i, d.max())
            assert abs(lse[h, i] - l) <= P.LSE_ABS, (h, i)
