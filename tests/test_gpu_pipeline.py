"""GPU parity of the whole forward path (layout -> reorder -> predict ->
attention -> inverse reorder) against the oracle, on the toy ledger and on
sampled rows of the image and video workloads at full size."""

import math

import numpy as np
import pytest

from long_context_mean_b200 import inputs as I
from oracle import attention as A
from oracle import layout as Y
from oracle import predict as Pr
from tests import _parity as P

pytestmark = pytest.mark.gpu


def run_pipeline(w, g, flags=0):
    from long_context_mean_b200 import sa
    q, k, v = P.qkv_dev(g, w.dtype)
    pipe = sa.pipeline_for(w, flags=flags, log_skips=True)
    out, lse = pipe.run(q, k, v)
    st = pipe.status()
    return pipe, out.float().cpu().numpy(), lse.cpu().numpy()[..., 0], st


def oracle_check(w, g, pipe, out, lse, heads, qblocks):
    """Oracle on the permuted inputs with the GPU's mask (validated against
    the oracle's own mask up to the boundary bands first)."""
    perm, inv = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    q, k, v = (Y.reorder(g[n], perm) for n in "qkv")
    B, Hq = w.B, w.Hq
    nqb, nkb = pipe.mask.struct.nqb, pipe.mask.struct.nkb
    gmask = pipe.mask.block_mask.cpu().numpy().reshape(B, Hq, nqb, nkb).astype(bool)
    orc = Pr.predict_mask(q, k, w.bq, w.bk, w.tau, w.theta, w.causal, w.sink_tokens, w.txt_len,
                          w.local_window, w.anchor_tokens)
    P.compare_masks(gmask, orc, w.tau, w.theta, w.Hq // w.Hkv)
    ref = A.block_sparse_attention_heads(q, k, v, gmask, w.bq, w.bk, w.causal, w.lam, heads=heads,
                                         qblocks=qblocks)
    if w.lam > -math.inf:
        rp = pipe.mask.row_ptr.cpu().numpy()
        ci = pipe.mask.col_idx.cpu().numpy()
        over = P.skip_override_from_gpu(pipe.skip_log.cpu().numpy(), rp, ci, nqb, B, Hq)
        if P.check_skip_decisions(over, ref["skips"], ref["gaps"], w.lam):
            ref = A.block_sparse_attention_heads(q, k, v, gmask, w.bq, w.bk, w.causal, w.lam, heads=heads,
                                                 qblocks=qblocks, skip_override=over, band=P.LAMBDA_BAND)
    # back to the original token order
    ref_out = Y.unreorder(ref["out"], perm, axis=2)
    ref_lse = Y.unreorder(ref["lse"], perm, axis=2)
    return P.attention_check(out, lse, {"out": ref_out, "lse": ref_lse}, label=f"{w.name} pipeline")


def dense_lse_gpu(w, g):
    """LSE of dense attention (sa_dense_attn) on the original-order inputs:
    dense attention is permutation-equivariant, so its rows line up with the
    pipeline's original-order LSE."""
    import torch
    from long_context_mean_b200 import sa
    q, k, v = P.qkv_dev(g, w.dtype)
    shape = sa.make_shape(q, k, v)
    out = torch.empty((w.B, w.Hq, w.N, w.dv), dtype=q.dtype, device="cuda")
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.dense_attn(q, k, v, shape, w.causal, 0.0, out, lse, st)
    assert sa.read_status(st) == sa.SA_OK
    return lse.cpu().numpy()


@pytest.mark.parametrize("flags", [0, 1])
def test_toy_pipeline(flags):
    w = I.WORKLOADS["toy"]
    g = I.gen_qkv(w)
    pipe, out, lse, st = run_pipeline(w, g, flags)
    assert st == 0
    oracle_check(w, g, pipe, out, lse, None, None)
    # dropped mass of every row against the oracle's dense attention
    dense = np.stack([[A.dense_attention(g["q"][b, h], g["k"][b, h], g["v"][b, h], w.causal)[1]
                       for h in range(w.Hq)] for b in range(w.B)])
    P.alpha_report(f"toy pipeline flags={flags}", lse, dense)


def test_toy_full_and_same_frame_masks():
    """The worked example's fixed masks on the toy grid: full and same-frame
    (block-diagonal 16-token blocks) through sa_mask_from_blocks."""
    import torch
    from long_context_mean_b200 import sa
    w = I.WORKLOADS["toy"]
    g = I.gen_qkv(w)
    q, k, v = P.qkv_dev(g, "fp32")
    shape = sa.make_shape(q, k, v)
    for name, blocks in (("full", np.ones((4, 4), bool)), ("spatial", np.eye(4, dtype=bool))):
        mb = sa.MaskBuffers.allocate(1, 1, 64, 16, 16, "cuda")
        ws = sa.workspace(sa.mask_from_blocks_workspace(shape, 16, 16), "cuda")
        sa.mask_from_blocks(torch.from_numpy(blocks.astype(np.uint8).ravel()).cuda(), shape, 16, 16, False,
                            ws, mb.struct)
        out = torch.empty_like(q)
        lse = torch.empty(1, 1, 64, dtype=torch.float32, device="cuda")
        sa.block_sparse_attn(q, k, v, shape, mb.struct, -math.inf, 0.0, out, lse)
        assert sa.read_status(mb.status) == 0
        tok = A.kept_blocks_to_token_mask(blocks, 64, 16, 16)
        y, _, l = A.masked_attention(g["q"][0, 0], g["k"][0, 0], g["v"][0, 0], tok)
        assert np.abs(out.cpu().numpy()[0, 0] - y).max() < 1e-5
        assert np.abs(lse.cpu().numpy()[0, 0] - l).max() < 1e-5


def gpu_block_sparsity(w, pipe):
    """1 - kept / causally valid tiles of the GPU's mask, over batch and heads."""
    nqb, nkb = pipe.mask.struct.nqb, pipe.mask.struct.nkb
    kept = int(pipe.mask.row_ptr.cpu().numpy()[-1])
    if w.causal:
        valid = w.B * w.Hq * sum(min(nkb, (min(w.N, (qb + 1) * w.bq) - 1) // w.bk + 1) for qb in range(nqb))
    else:
        valid = w.B * w.Hq * nqb * nkb
    return 1.0 - kept / valid


def test_toy_same_position_mask_through_the_window_reorder():
    """The toy grid's third fixed mask ([P1] 3.3: each token with the same
    pixel in every frame, 256 pairs): the [T,1,1] window layout puts a pixel's
    frames next to each other ([P1] 3.4, token-major order), where the mask is
    block-diagonal with 4-token blocks (bq = bk = 4, 16 of 256 tiles).  Layout,
    reorder, attention and inverse reorder run on the GPU; the oracle applies
    the element mask in the original order."""
    import torch
    from long_context_mean_b200 import sa
    from oracle import ledger as L
    w = I.WORKLOADS["toy"]
    g = I.gen_qkv(w)
    q, k, v = P.qkv_dev(g, "fp32")
    lay = sa.make_layout(4, 4, 4, 0, 0, "window", (4, 1, 1))
    perm = torch.empty(64, dtype=torch.int32, device="cuda")
    inv = torch.empty_like(perm)
    sa.layout_build(lay, perm, inv)
    ref_perm, _ = Y.build_layout("window", 4, 4, 4, (4, 1, 1), 0, 0)
    assert np.array_equal(perm.cpu().numpy(), ref_perm)
    qr, kr, vr = (torch.empty_like(x) for x in (q, k, v))
    for x, y in ((q, qr), (k, kr), (v, vr)):
        sa.reorder(perm, x, y)
    shape = sa.make_shape(q, k, v)
    blocks = np.eye(16, dtype=bool)
    mb = sa.MaskBuffers.allocate(1, 1, 64, 4, 4, "cuda")
    ws = sa.workspace(sa.mask_from_blocks_workspace(shape, 4, 4), "cuda")
    sa.mask_from_blocks(torch.from_numpy(blocks.astype(np.uint8).ravel()).cuda(), shape, 4, 4, False, ws,
                        mb.struct)
    out = torch.empty_like(q)
    lse = torch.empty(1, 1, 64, 1, dtype=torch.float32, device="cuda")
    sa.block_sparse_attn(qr, kr, vr, shape, mb.struct, -math.inf, 0.0, out, lse, out_perm=perm)
    assert sa.read_status(mb.status) == 0
    assert int(mb.kept_total.item()) == 16
    tok = L.video_masks(4, 4, 4)["temporal"]
    assert int(tok.sum()) == 256
    y, _, l = A.masked_attention(g["q"][0, 0], g["k"][0, 0], g["v"][0, 0], tok)
    assert np.abs(out.cpu().numpy()[0, 0] - y).max() < 1e-5
    assert np.abs(lse.cpu().numpy()[0, 0, :, 0] - l).max() < 1e-5


@pytest.mark.parametrize("name", ["video", "image", "image_s60"])
def test_full_size_pipeline_sampled(name):
    w = I.WORKLOADS[name]
    g = I.gen_qkv(w)
    pipe, out, lse, st = run_pipeline(w, g)
    assert st == 0
    if w.theta <= 0 and w.target_sparsity > 0:
        s = gpu_block_sparsity(w, pipe)
        P.report(f"{name} block sparsity", sparsity=s, target=w.target_sparsity)
        assert abs(s - w.target_sparsity) <= 0.01
    nqb = pipe.mask.struct.nqb
    heads = [(0, 0), (0, w.Hq - 1)] + ([(1, 5)] if w.B > 1 else [(0, 7)])
    qblocks = sorted({0, 1, nqb // 2, nqb - 2, nqb - 1})
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    rows = np.zeros(w.N, bool)
    for qb in qblocks:
        rows[qb * w.bq:(qb + 1) * w.bq] = True
    rows_orig = np.zeros(w.N, bool)
    rows_orig[perm[rows]] = True
    sel = np.zeros((w.B, w.Hq, w.N), bool)
    for b, h in heads:
        sel[b, h] = rows_orig
    oracle_check(w, g, pipe, out, lse, heads, qblocks)
    P.alpha_report(f"{name} pipeline, every row", lse, dense_lse_gpu(w, g))


def _sampled_heads_check(w, heads, kv_of, qblocks):
    """Full-size run of the whole path; the oracle recomputes the mask and the
    attention for the listed (b, h) heads and q-blocks only."""
    import torch
    from long_context_mean_b200 import sa
    g = I.gen_qkv(w)
    q, k, v = P.qkv_dev(g, w.dtype)
    pipe = sa.pipeline_for(w, log_skips=True)
    out, lse = pipe.run(q, k, v)
    assert pipe.status() == 0
    out_h = out.float().cpu().numpy()
    lse_h = lse.cpu().numpy()[..., 0]
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    nqb, nkb = pipe.mask.struct.nqb, pipe.mask.struct.nkb
    gmask = pipe.mask.block_mask.cpu().numpy().reshape(w.B, w.Hq, nqb, nkb).astype(bool)
    rp = pipe.mask.row_ptr.cpu().numpy()
    ci = pipe.mask.col_idx.cpu().numpy()
    skip = pipe.skip_log.cpu().numpy()
    for b, h in heads:
        g_h = kv_of(h)
        qh = Y.reorder(g["q"][b:b + 1, h:h + 1], perm)
        kh = Y.reorder(g["k"][b:b + 1, g_h:g_h + 1], perm)
        vh = Y.reorder(g["v"][b:b + 1, g_h:g_h + 1], perm)
        orc = Pr.predict_mask(qh, kh, w.bq, w.bk, w.tau, w.theta, w.causal, w.sink_tokens, w.txt_len,
                              w.local_window, w.anchor_tokens)
        P.compare_masks(gmask[b:b + 1, h:h + 1], orc, w.tau, w.theta, 1)
        m = gmask[b:b + 1, h:h + 1]
        ref = A.block_sparse_attention_heads(qh, kh, vh, m, w.bq, w.bk, w.causal, w.lam, qblocks=qblocks)
        if w.lam > -math.inf:
            over = {}
            base = (b * w.Hq + h) * nqb
            for qb in qblocks:
                u = base + qb
                for t in range(rp[u], rp[u + 1]):
                    over[(0, 0, qb, int(ci[t]))] = bool(skip[t])
            if P.check_skip_decisions(over, ref["skips"], ref["gaps"], w.lam):
                ref = A.block_sparse_attention_heads(qh, kh, vh, m, w.bq, w.bk, w.causal, w.lam, qblocks=qblocks,
                                                     skip_override=over, band=P.LAMBDA_BAND)
        ref_out = Y.unreorder(ref["out"], perm, axis=2)
        ref_lse = Y.unreorder(ref["lse"], perm, axis=2)
        P.attention_check(out_h[b:b + 1, h:h + 1], lse_h[b:b + 1, h:h + 1], {"out": ref_out, "lse": ref_lse},
                          label=f"{w.name} sampled head ({b},{h})")
    P.alpha_report(f"{w.name} pipeline, every row", lse_h, dense_lse_gpu(w, g))
    return pipe


def test_video_large_hilbert_sampled():
    w = I.WORKLOADS["video_large"]
    nqb = -(-w.N // w.bq)
    _sampled_heads_check(w, [(0, 0), (0, 23)], lambda h: h, [0, 300, nqb - 1])


def test_video_large_hilbert_at_sparsity_085_sampled():
    """The large Hilbert video at its stated block sparsity (guard off):
    TopCdf, the ragged lists and the scheduler do real work at this size."""
    w = I.WORKLOADS["video_large_s85"]
    nqb = -(-w.N // w.bq)
    pipe = _sampled_heads_check(w, [(0, 0), (0, 11), (0, 23)], lambda h: h, [0, 29, 300, 411, nqb - 1])
    s = gpu_block_sparsity(w, pipe)
    P.report("video_large_s85 block sparsity", sparsity=s, target=w.target_sparsity)
    assert abs(s - w.target_sparsity) <= 0.01


def test_lm_causal_gqa_sampled():
    """The causal 131K GQA workload: whole-head masks for four heads (KV heads
    0, 2, 4 and 7), attention on seven query blocks of each, and the grouped
    work order of all 32,768 rows bit-exact against the oracle's."""
    w = I.WORKLOADS["lm_causal"]
    nqb = -(-w.N // w.bq)
    pipe = _sampled_heads_check(w, [(0, 0), (0, 9), (0, 18), (0, 29)], lambda h: h // (w.Hq // w.Hkv),
                                [0, 1, 40, 255, 513, 800, nqb - 1])
    G = int(pipe.params.order_group)
    assert G == 4
    gmask = pipe.mask.block_mask.cpu().numpy().reshape(w.B, w.Hq, nqb, -1).astype(bool)
    assert np.array_equal(pipe.mask.order.cpu().numpy(), Pr.mask_to_csr(gmask, G)["order"])


@pytest.mark.parametrize("name,chunks", [("video", 4), ("lm_small", 2)])
def test_host_pipeline_matches_device_pipeline(name, chunks):
    """The chunked host-to-host pass (copies overlapped with the kernels)
    returns exactly what the device pipeline computes: heads are independent
    and every chunk runs the same kernels on its rows."""
    import torch
    from long_context_mean_b200 import sa
    if name == "lm_small":
        w = I.Workload("lm_small", 55, 2, 4, 2, 1, 1, 1500, 0, 128, 128, "bf16", "lowrank", bq=128, bk=64,
                       tau=0.9, causal=True, local_window=300, anchor_tokens=64, sigma_pos=40.0)
    else:
        w = I.WORKLOADS[name]
    g = I.gen_qkv(w)
    host = {n: torch.from_numpy(g[n + "_bits"].view(np.int16)).view(torch.bfloat16).pin_memory() for n in "qkv"}
    q, k, v = (host[n].to("cuda") for n in "qkv")
    pipe = sa.pipeline_for(w)
    out_d, lse_d = pipe.run(q, k, v)
    assert pipe.status() == sa.SA_OK
    hp = sa.host_pipeline_for(w, chunks=chunks)
    out_h = torch.empty(out_d.shape, dtype=out_d.dtype).pin_memory()
    lse_h = torch.empty(lse_d.shape, dtype=lse_d.dtype).pin_memory()
    for _ in range(2):                  # twice: the second pass reuses every buffer
        out_h.fill_(0)
        lse_h.fill_(0)
        hp.run(host["q"], host["k"], host["v"], out_h, lse_h)
        hp.done.synchronize()
        assert hp.status() == sa.SA_OK
        assert torch.equal(out_h, out_d.cpu())
        assert torch.equal(lse_h, lse_d.cpu())


@pytest.mark.parametrize("name", ["fused_window", "toy_identity"])
def test_graph_replay_matches_eager_run(name):
    """Pipeline.capture/replay: the whole path (side stream included) as one
    CUDA graph gives the eager run's outputs bit for bit, and a replay after
    new inputs are written in place gives the eager outputs for those."""
    import torch
    from long_context_mean_b200 import sa
    if name == "fused_window":
        w = I.Workload("fused_window", 77, 1, 4, 4, 5, 12, 20, 37, 128, 128, "bf16", "field", order="window",
                       win=(2, 8, 8), sink_frames=1, bq=128, bk=64, tau=0.5, theta=0.0, lam=-5.0,
                       sigma=(1.0, 2.0, 2.0))
    else:
        w = I.Workload("toy_identity", 78, 1, 2, 1, 1, 1, 1500, 0, 128, 128, "bf16", "lowrank", bq=128, bk=64,
                       tau=0.8, causal=True, local_window=256, anchor_tokens=64)
    g1, g2 = I.gen_qkv(w), I.gen_qkv(I.Workload(**{**w.__dict__, "seed": w.seed + 1}))
    q, k, v = P.qkv_dev(g1, w.dtype)
    q2, k2, v2 = P.qkv_dev(g2, w.dtype)
    eager = sa.pipeline_for(w)
    out_e, lse_e = (x.clone() for x in eager.run(q, k, v))
    out_e2, lse_e2 = (x.clone() for x in eager.run(q2, k2, v2))
    assert eager.status() == sa.SA_OK
    pipe = sa.pipeline_for(w)
    pipe.capture(q, k, v)
    out, lse = pipe.replay()
    torch.cuda.synchronize()
    assert pipe.status() == sa.SA_OK
    assert torch.equal(out, out_e) and torch.equal(lse, lse_e)
    q.copy_(q2)
    k.copy_(k2)
    v.copy_(v2)
    out, lse = pipe.replay()
    torch.cuda.synchronize()
    assert pipe.status() == sa.SA_OK
    assert torch.equal(out, out_e2) and torch.equal(lse, lse_e2)
