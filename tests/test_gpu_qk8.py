"""GPU parity of the 8-bit QK paths, INT8 and FP8 E4M3 (sa_quantize_blocks,
sa_block_sparse_attn_qk8 and Pipeline(qk8=...)) against oracle.quant."""

import math

import numpy as np
import pytest

from long_context_mean_b200 import inputs as I
from oracle import layout as Y
from oracle import predict as Pr
from oracle import quant as Q
from tests import _parity as P
from tests.test_gpu_attention import random_mask

pytestmark = pytest.mark.gpu


FORMATS = ["int8", "e4m3"]


def _quantize_dev(xd, rows, fmt):
    import torch
    from long_context_mean_b200 import sa
    N = xd.shape[-2]
    heads = xd.numel() // (N * xd.shape[-1])
    x8 = torch.empty(xd.shape, dtype=torch.uint8, device="cuda")
    sc = torch.empty(heads * (-(-N // rows)), dtype=torch.float32, device="cuda")
    sa.quantize_blocks(xd, rows, x8, sc, fmt)
    return x8, sc


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("rows", [128, 64, 1])
def test_quantize_blocks_bit_exact(rows, fmt):
    rng = np.random.default_rng(rows)
    x = (rng.standard_normal((2, 3, 300, 128)) * rng.uniform(0.01, 20, size=(2, 3, 300, 1))).astype(np.float32)
    x[0, 1, :rows] = 0.0                       # an all-zero block
    x[1, 2, 5, 7] = 1e-38                      # a subnormal-range value
    x[1, 0, 3, :4] = [-0.0, 1e-30, -1e-30, 3.0]   # signed zero and codes that round to zero
    bits = I.to_bf16_bits(x)
    x8, sc = _quantize_dev(P.bf16_dev(bits), rows, fmt)
    ref8, refs = Q.quantize_blocks(I.bf16_bits_to_f32(bits), rows, fmt)
    assert np.array_equal(x8.cpu().numpy().view(ref8.dtype), ref8)
    assert np.array_equal(sc.cpu().numpy().reshape(refs.shape).view(np.uint32), refs.view(np.uint32))


def _run_qk8(qd, kd, vd, m, bq, bk, lam, fmt, flags=0):
    import torch
    from long_context_mean_b200 import sa
    shape = sa.make_shape(qd, kd, vd)
    B, Hq, N = qd.shape[:3]
    mb = sa.MaskBuffers.allocate(B, Hq, N, bq, bk, "cuda")
    ws = sa.workspace(sa.mask_from_blocks_workspace(shape, bq, bk), "cuda")
    sa.mask_from_blocks(torch.from_numpy(m.astype(np.uint8).ravel()).cuda(), shape, bq, bk, False, ws, mb.struct)
    q8, qs = _quantize_dev(qd, bq, fmt)
    k8, ks = _quantize_dev(kd, bk, fmt)
    out = torch.full((B, Hq, N, vd.shape[3]), float("nan"), dtype=qd.dtype, device="cuda")
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    skip = torch.full((mb.col_idx.numel(),), 7, dtype=torch.uint8, device="cuda")
    aws = sa.workspace(sa.attn_qk8_workspace(mb.struct), "cuda")
    sa.block_sparse_attn_qk8(q8, qs, k8, ks, vd, shape, mb.struct, lam, 0.0, out, aws, lse, skip, flags, fmt=fmt)
    return {"status": sa.read_status(mb.status), "out": out.float().cpu().numpy(), "lse": lse.cpu().numpy(),
            "row_ptr": mb.row_ptr.cpu().numpy(), "col_idx": mb.col_idx.cpu().numpy(), "nqb": mb.struct.nqb,
            "skip": skip.cpu().numpy()}


QK8_CASES = [
    # name, B, Hq, Hkv, N, bk, lam, p
    ("bk64", 1, 3, 3, 700, 64, -math.inf, 0.5),
    ("bk64_lam_gqa", 1, 4, 2, 900, 64, -3.0, 0.6),
    ("bk128", 1, 2, 2, 650, 128, -math.inf, 0.5),
    ("bk64_dense_mask", 2, 2, 2, 1024, 64, -math.inf, 1.0),
]


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("case", QK8_CASES, ids=[c[0] for c in QK8_CASES])
def test_qk8_attention_vs_oracle(case, fmt):
    name, B, Hq, Hkv, N, bk, lam, p = case
    rng = np.random.default_rng(len(name) * 17 + N)
    w = I.Workload(name, 700 + N, B, Hq, Hkv, 1, 1, N, 0, 128, 128, "bf16", "field" if Hq == Hkv else "lowrank",
                   sigma=(0.0, 0.0, 8.0), sigma_pos=30.0, noise=0.5)
    g = I.gen_qkv(w)
    qd, kd, vd = P.qkv_dev(g, "bf16")
    m = random_mask(rng, B, Hq, N, 128, bk, False, p)
    r = _run_qk8(qd, kd, vd, m, 128, bk, lam, fmt)
    assert r["status"] == 0
    ref = Q.block_sparse_attention_qk8_heads(g["q"], g["k"], g["v"], m, 128, bk, False, lam, fmt=fmt)
    if lam > -math.inf:
        over = P.skip_override_from_gpu(r["skip"], r["row_ptr"], r["col_idx"], r["nqb"], B, Hq)
        if P.check_skip_decisions(over, ref["skips"], ref["gaps"], lam):
            ref = Q.block_sparse_attention_qk8_heads(g["q"], g["k"], g["v"], m, 128, bk, False, lam,
                                                     skip_override=over, band=P.LAMBDA_BAND, fmt=fmt)
    P.attention_check(r["out"], r["lse"], ref)


def test_qk8_rejects_the_simt_flag():
    import torch
    from long_context_mean_b200 import sa
    w = I.Workload("rej", 11, 1, 1, 1, 1, 1, 256, 0, 128, 128, "bf16", "iid")
    g = I.gen_qkv(w)
    qd, kd, vd = P.qkv_dev(g, "bf16")
    with pytest.raises(sa.SAError) as e:
        _run_qk8(qd, kd, vd, np.ones((1, 1, 2, 4), bool), 128, 64, -math.inf, "int8", flags=1)
    assert e.value.code == sa.SA_ERR_UNSUPPORTED


@pytest.mark.parametrize("fmt", FORMATS)
def test_pipeline_qk8_video_sampled(fmt):
    """The video workload through Pipeline(qk8=True): the mask is the bf16
    prediction's, the attention the quantised one; sampled heads and query
    blocks against the oracle on the permuted inputs."""
    from long_context_mean_b200 import sa
    w = I.WORKLOADS["video"]
    g = I.gen_qkv(w)
    q, k, v = P.qkv_dev(g, w.dtype)
    pipe = sa.pipeline_for(w, log_skips=True, qk8=fmt)
    out, lse = pipe.run(q, k, v)
    assert pipe.status() == 0
    out = out.float().cpu().numpy()
    lse = lse.cpu().numpy()[..., 0]
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    nqb, nkb = pipe.mask.struct.nqb, pipe.mask.struct.nkb
    gmask = pipe.mask.block_mask.cpu().numpy().reshape(w.B, w.Hq, nqb, nkb).astype(bool)
    rp = pipe.mask.row_ptr.cpu().numpy()
    ci = pipe.mask.col_idx.cpu().numpy()
    skip = pipe.skip_log.cpu().numpy()
    qblocks = sorted({0, 1, nqb // 2, nqb - 1})
    for h in (0, 13, w.Hq - 1):
        qh, kh, vh = (Y.reorder(g[n][:, h:h + 1], perm) for n in "qkv")
        orc = Pr.predict_mask(qh, kh, w.bq, w.bk, w.tau, w.theta, w.causal, w.sink_tokens, w.txt_len,
                              w.local_window, w.anchor_tokens)
        P.compare_masks(gmask[:, h:h + 1], orc, w.tau, w.theta, 1)
        m = gmask[:, h:h + 1]
        over = {}
        for qb in qblocks:
            u = h * nqb + qb
            for t in range(rp[u], rp[u + 1]):
                over[(0, 0, qb, int(ci[t]))] = bool(skip[t])
        ref = Q.block_sparse_attention_qk8_heads(qh, kh, vh, m, w.bq, w.bk, False, w.lam, qblocks=qblocks,
                                                 fmt=fmt)
        if P.check_skip_decisions(over, ref["skips"], ref["gaps"], w.lam):
            ref = Q.block_sparse_attention_qk8_heads(qh, kh, vh, m, w.bq, w.bk, False, w.lam, qblocks=qblocks,
                                                     skip_override=over, band=P.LAMBDA_BAND, fmt=fmt)
        ref_out = Y.unreorder(ref["out"], perm, axis=2)
        ref_lse = Y.unreorder(ref["lse"], perm, axis=2)
        P.attention_check(out[:, h:h + 1], lse[:, h:h + 1], {"out": ref_out, "lse": ref_lse})


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("reordered", [True, False])
def test_fused_codes_match_quantised_reordered_inputs(fmt, reordered):
    """sa_reorder_predict_mask_q8 on the video workload: the codes and scales
    its pooling pass writes equal the oracle's quantisation of the reordered
    (or original) Q and K, and the mask equals the bf16 prediction's."""
    import torch
    from long_context_mean_b200 import sa
    w = I.WORKLOADS["video"]
    g = I.gen_qkv(w)
    q, k, v = P.qkv_dev(g, w.dtype)
    pipe = sa.pipeline_for(w)
    shape = pipe.shape
    if reordered:
        sa.layout_build(pipe.layout, pipe.perm, pipe.inv, pipe.layout_ws)
        perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
        assert np.array_equal(pipe.perm.cpu().numpy(), perm)
        perm_dev = pipe.perm
    else:
        perm_dev, perm = None, np.arange(w.N)
    nqb, nkb = pipe.mask.struct.nqb, pipe.mask.struct.nkb
    q8 = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
    k8 = torch.empty(k.shape, dtype=torch.uint8, device="cuda")
    qs = torch.empty(w.B * w.Hq * nqb, dtype=torch.float32, device="cuda")
    ks = torch.empty(w.B * w.Hkv * nkb, dtype=torch.float32, device="cuda")
    m8 = sa.MaskBuffers.allocate(w.B, w.Hq, w.N, w.bq, w.bk, "cuda")
    sa.reorder_predict_mask_q8(perm_dev, q, k, fmt, q8, qs, k8, ks, shape, pipe.params, pipe.ws, m8.struct)
    assert sa.read_status(m8.status) == 0
    qr = torch.empty_like(q)
    kr = torch.empty_like(k)
    mb = sa.MaskBuffers.allocate(w.B, w.Hq, w.N, w.bq, w.bk, "cuda")
    if reordered:
        sa.reorder_predict_mask(pipe.perm, q, k, qr, kr, shape, pipe.params, pipe.ws, mb.struct)
    else:
        sa.predict_mask(q, k, shape, pipe.params, pipe.ws, mb.struct)
    assert sa.read_status(mb.status) == 0
    assert torch.equal(m8.block_mask, mb.block_mask)
    for x8, sc, name, rows in ((q8, qs, "q", w.bq), (k8, ks, "k", w.bk)):
        ref8, refs = Q.quantize_blocks(Y.reorder(g[name], perm), rows, fmt)
        assert np.array_equal(x8.cpu().numpy().view(ref8.dtype), ref8)
        assert np.array_equal(sc.cpu().numpy().reshape(refs.shape).view(np.uint32), refs.view(np.uint32))
