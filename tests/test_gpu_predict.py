"""GPU parity: mask prediction (pooling, similarity guard, TopCdf, forced
blocks) and the CSR lists / work order, against the fp64 oracle."""

import math

import numpy as np
import pytest

from long_context_mean_b200 import inputs as I
from oracle import layout as Y
from oracle import predict as Pr
from tests import _parity as P

pytestmark = pytest.mark.gpu


def run_gpu_predict(q_dev, k_dev, w, params, capacity=None):
    import torch
    from long_context_mean_b200 import sa
    shape = sa.Shape(q_dev.shape[0], q_dev.shape[1], k_dev.shape[1], q_dev.shape[2], q_dev.shape[3],
                     q_dev.shape[3], sa.dtype_code(q_dev), 0)
    ws = sa.workspace(sa.predict_mask_workspace(shape, params), "cuda")
    ws.fill_(0xFF)          # poison: every output must be written
    mb = sa.MaskBuffers.allocate(shape.B, shape.Hq, shape.N, params.bq, params.bk, "cuda", capacity)
    mb.row_ptr.fill_(-7)
    mb.order.fill_(-7)
    sa.predict_mask(q_dev, k_dev, shape, params, ws, mb.struct)
    status = sa.read_status(mb.status)
    off = sa.predict_mask_ws_layout(shape, params)
    nqb, nkb = mb.struct.nqb, mb.struct.nkb
    B, Hq, Hkv, d = shape.B, shape.Hq, shape.Hkv, shape.d

    def view(i, n):
        return ws[off[i]:off[i] + n * 4].view(torch.float32).cpu().numpy()
    out = {
        "status": status,
        "qhat": view(0, B * Hq * nqb * d).reshape(B, Hq, nqb, d),
        "khat": khat_from_ws(ws, off, B, Hkv, nkb, d),
        "s_q": view(2, B * Hq * nqb).reshape(B, Hq, nqb),
        "s_k": view(3, B * Hkv * nkb).reshape(B, Hkv, nkb),
        "mask": mb.block_mask.cpu().numpy().reshape(B, Hq, nqb, nkb).astype(bool),
        "row_ptr": mb.row_ptr.cpu().numpy(),
        "col_idx": mb.col_idx.cpu().numpy(),
        "order": mb.order.cpu().numpy(),
        "kept_total": int(mb.kept_total.item()),
    }
    return out


def khat_from_ws(ws, off, B, Hkv, nkb, d):
    """k_hat from the prediction workspace, stored feature-major [B*Hkv, d, nkb4]."""
    import torch
    nkb4 = (nkb + 3) // 4 * 4
    kt = ws[off[1]:off[1] + B * Hkv * d * nkb4 * 4].view(torch.float32).cpu().numpy()
    return np.ascontiguousarray(kt.reshape(B, Hkv, d, nkb4)[..., :nkb].swapaxes(-1, -2))


def oracle_predict(q, k, w):
    return Pr.predict_mask(q, k, w.bq, w.bk, w.tau, w.theta, w.causal, w.sink_tokens, w.txt_len,
                           w.local_window, w.anchor_tokens)


def check_lists(g, mask, order_group=0):
    c = Pr.mask_to_csr(mask, order_group)
    assert g["kept_total"] == c["kept_total"]
    assert np.array_equal(g["row_ptr"], c["row_ptr"])
    assert np.array_equal(g["col_idx"][:c["kept_total"]], c["col_idx"])
    assert np.array_equal(g["order"], c["order"])


def check_predict(w, q_np, k_np, q_dev, k_dev):
    from long_context_mean_b200 import sa
    prm = sa.make_params(w.bq, w.bk, w.tau, w.theta, w.sink_tokens, w.txt_len, w.local_window,
                         w.anchor_tokens, w.causal)
    g = run_gpu_predict(q_dev, k_dev, w, prm)
    assert g["status"] == sa.SA_OK
    orc = oracle_predict(q_np, k_np, w)
    np.testing.assert_allclose(g["qhat"], orc["qhat"], rtol=0, atol=2e-6 * max(1, np.abs(orc["qhat"]).max()))
    np.testing.assert_allclose(g["khat"], orc["khat"], rtol=0, atol=2e-6 * max(1, np.abs(orc["khat"]).max()))
    np.testing.assert_allclose(g["s_q"], orc["s_q"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(g["s_k"], orc["s_k"], rtol=0, atol=2e-6)
    ndiff = P.compare_masks(g["mask"], orc, w.tau, w.theta, w.Hq // w.Hkv)
    # The lists are a function of the mask: bit-exact against the oracle's
    # compaction of the GPU's mask (identical to the oracle's own mask when
    # no boundary block differs).
    check_lists(g, g["mask"])
    if ndiff == 0:
        check_lists(g, orc["mask"])
    return g, orc, ndiff


SMALL = [
    # name, B, Hq, Hkv, N, d, bq, bk, tau, theta, causal, sink, txt, window, anchors, dtype
    ("plain", 1, 2, 2, 700, 64, 64, 32, 0.6, 0.0, False, 0, 0, 0, 0, "bf16"),
    ("guard", 2, 3, 3, 513, 128, 128, 64, 0.5, 0.25, False, 0, 0, 0, 0, "bf16"),
    ("sink_text", 1, 2, 2, 1000, 128, 128, 64, 0.3, 0.0, False, 130, 77, 0, 0, "bf16"),
    ("causal_gqa", 1, 4, 2, 1500, 128, 128, 64, 0.8, 0.0, True, 0, 0, 300, 128, "bf16"),
    ("causal_small_blocks", 1, 2, 1, 333, 32, 16, 8, 0.9, 0.0, True, 0, 0, 40, 5, "fp32"),
    ("toy", 1, 1, 1, 64, 16, 16, 16, 0.9, 0.5, False, 0, 0, 0, 0, "fp32"),
    ("tau_one", 1, 2, 2, 640, 128, 128, 64, 1.0, 0.0, False, 0, 0, 0, 0, "bf16"),
    # more than 512 key blocks: TopCdf's threshold search instead of the arg-max loop
    ("threshold_search", 1, 2, 2, 6000, 64, 32, 8, 0.9, 0.0, False, 0, 0, 0, 0, "bf16"),
    ("threshold_causal", 1, 2, 1, 6000, 64, 32, 8, 0.95, 0.0, True, 0, 0, 64, 8, "bf16"),
    ("threshold_low_tau", 1, 2, 2, 6000, 64, 32, 8, 0.25, 0.0, False, 0, 0, 0, 0, "bf16"),
    # above tau = 0.999 the threshold search starts at 0 (no lower start)
    ("threshold_near_one", 1, 2, 2, 6000, 64, 32, 8, 0.9995, 0.0, False, 0, 0, 0, 0, "bf16"),
    # 2048 key blocks: the scores of four consecutive blocks per thread
    ("long_rows", 1, 2, 1, 16384, 32, 64, 8, 0.9, 0.0, True, 0, 0, 128, 16, "bf16"),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_predict_small(case):
    name, B, Hq, Hkv, N, d, bq, bk, tau, theta, causal, sink, txt, win, anch, dt = case
    w = I.Workload(name, 77 + len(name), B, Hq, Hkv, 1, 1, N - txt, txt, d, d, dt, "field" if Hq == Hkv else "lowrank",
                   bq=bq, bk=bk, tau=tau, theta=theta, causal=causal, local_window=win,
                   anchor_tokens=anch, sigma=(0.0, 0.0, 6.0), sigma_pos=20.0)
    g = I.gen_qkv(w)
    q_dev, k_dev, _ = P.qkv_dev(g, dt)
    # sink tokens are given directly for these synthetic cases
    from long_context_mean_b200 import sa
    prm = sa.make_params(bq, bk, tau, theta, sink, txt, win, anch, causal)
    gres = run_gpu_predict(q_dev, k_dev, w, prm)
    assert gres["status"] == sa.SA_OK
    orc = Pr.predict_mask(g["q"], g["k"], bq, bk, tau, theta, causal, sink, txt, win, anch)
    np.testing.assert_allclose(gres["s_q"], orc["s_q"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(gres["s_k"], orc["s_k"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(gres["qhat"], orc["qhat"], rtol=0, atol=1e-5)
    P.compare_masks(gres["mask"], orc, tau, theta, Hq // Hkv)
    check_lists(gres, gres["mask"])
    assert gres["mask"].any()


@pytest.mark.parametrize("name", ["video", "image"])
def test_predict_full_size(name):
    w = I.WORKLOADS[name]
    g = I.gen_qkv(w)
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    qn, kn = Y.reorder(g["q"], perm), Y.reorder(g["k"], perm)
    import torch
    q_dev = P.bf16_dev(Y.reorder(g["q_bits"], perm))
    k_dev = P.bf16_dev(Y.reorder(g["k_bits"], perm))
    gres, orc, ndiff = check_predict(w, qn, kn, q_dev, k_dev)
    valid = np.broadcast_to(orc["valid"][:, None], gres["mask"].shape)
    sp = Pr.block_sparsity(gres["mask"], valid)
    if name == "video":
        assert abs(sp - w.target_sparsity) < 0.01
    else:
        assert sp == 0.0     # theta = 0.6 forces every block of this generator


@pytest.mark.parametrize("order_group", [1, 2, 3])
def test_work_order_in_head_groups(order_group):
    """order_group > 0: the work order sorts each group of consecutive
    (batch, head) rows on its own, bit-exact against the oracle's order."""
    from long_context_mean_b200 import sa
    B, Hq, Hkv, N, bq, bk = 2, 4, 2, 1500, 128, 64
    w = I.Workload("groups", 99, B, Hq, Hkv, 1, 1, N, 0, 128, 128, "bf16", "lowrank", bq=bq, bk=bk, tau=0.8,
                   causal=True, local_window=300, anchor_tokens=128, sigma_pos=20.0)
    g = I.gen_qkv(w)
    q_dev, k_dev, _ = P.qkv_dev(g, "bf16")
    prm = sa.make_params(bq, bk, 0.8, 0.0, 0, 0, 300, 128, True, order_group)
    gres = run_gpu_predict(q_dev, k_dev, w, prm)
    assert gres["status"] == sa.SA_OK
    check_lists(gres, gres["mask"], order_group)
    # the grouped order differs from the global one on this mask
    assert not np.array_equal(gres["order"], Pr.mask_to_csr(gres["mask"])["order"])


def test_global_order_past_shared_memory_rows():
    """More than 32768 rows: the work order comes from the global-memory
    radix sort, bit-exact against the oracle."""
    import torch
    from long_context_mean_b200 import sa
    rng = np.random.default_rng(11)
    B, Hq, bq, bk = 1, 40, 128, 128
    nqb = nkb = 1000
    N = nqb * bq
    dens = rng.random((B, Hq, nqb, 1)) * 0.6           # rows of many different lengths
    m = rng.random((B, Hq, nqb, nkb)) < dens
    m[..., 0] = True
    shape = sa.Shape(B, Hq, Hq, N, 128, 128, sa.SA_BF16, 0)
    blocks = torch.from_numpy(m.astype(np.uint8).ravel()).to("cuda")
    mb = sa.MaskBuffers.allocate(B, Hq, N, bq, bk, "cuda", capacity=int(m.sum()))
    ws = sa.workspace(sa.mask_from_blocks_workspace(shape, bq, bk), "cuda")
    sa.mask_from_blocks(blocks, shape, bq, bk, False, ws, mb.struct)
    assert sa.read_status(mb.status) == sa.SA_OK
    c = Pr.mask_to_csr(m)
    assert int(mb.kept_total.item()) == c["kept_total"]
    assert np.array_equal(mb.row_ptr.cpu().numpy(), c["row_ptr"])
    assert np.array_equal(mb.col_idx.cpu().numpy(), c["col_idx"])
    assert np.array_equal(mb.order.cpu().numpy(), c["order"])


def test_empty_row_status():
    import torch
    from long_context_mean_b200 import sa
    B, Hq, N, bq, bk = 1, 2, 256, 128, 64
    shape = sa.Shape(B, Hq, Hq, N, 128, 128, sa.SA_BF16, 0)
    nqb, nkb = 2, 4
    blocks = torch.ones(B * Hq * nqb * nkb, dtype=torch.uint8, device="cuda")
    blocks.view(B * Hq, nqb, nkb)[1, 1, :] = 0          # head 1, q-block 1: nothing kept
    mb = sa.MaskBuffers.allocate(B, Hq, N, bq, bk, "cuda")
    ws = sa.workspace(sa.mask_from_blocks_workspace(shape, bq, bk), "cuda")
    sa.mask_from_blocks(blocks, shape, bq, bk, False, ws, mb.struct)
    assert sa.read_status(mb.status) == sa.SA_ERR_EMPTY_ROW
    # causal: q-block 1 (rows 128..255) keeping only k-block 3 (keys 192..255)
    blocks.fill_(0)
    blocks.view(B * Hq, nqb, nkb)[:, 0, 0] = 1
    blocks.view(B * Hq, nqb, nkb)[:, 1, 3] = 1
    sa.mask_from_blocks(blocks, shape, bq, bk, True, ws, mb.struct)
    assert sa.read_status(mb.status) == sa.SA_ERR_EMPTY_ROW
    blocks.view(B * Hq, nqb, nkb)[:, 1, 2] = 1
    sa.mask_from_blocks(blocks, shape, bq, bk, True, ws, mb.struct)
    assert sa.read_status(mb.status) == sa.SA_OK


def test_capacity_status():
    import torch
    from long_context_mean_b200 import sa
    shape = sa.Shape(1, 1, 1, 512, 128, 128, sa.SA_BF16, 0)
    blocks = torch.ones(4 * 8, dtype=torch.uint8, device="cuda")
    mb = sa.MaskBuffers.allocate(1, 1, 512, 128, 64, "cuda", capacity=31)
    ws = sa.workspace(sa.mask_from_blocks_workspace(shape, 128, 64), "cuda")
    sa.mask_from_blocks(blocks, shape, 128, 64, False, ws, mb.struct)
    assert sa.read_status(mb.status) == sa.SA_ERR_CAPACITY


def test_mask_from_blocks_lists_and_causal_and():
    import torch
    from long_context_mean_b200 import sa
    rng = np.random.default_rng(3)
    B, Hq, N, bq, bk = 2, 3, 1000, 128, 64
    nqb, nkb = 8, 16
    m = rng.random((B, Hq, nqb, nkb)) < 0.3
    m[..., 0] = True
    shape = sa.Shape(B, Hq, Hq, N, 128, 128, sa.SA_BF16, 0)
    blocks = torch.from_numpy(m.astype(np.uint8).ravel()).to("cuda")
    mb = sa.MaskBuffers.allocate(B, Hq, N, bq, bk, "cuda")
    ws = sa.workspace(sa.mask_from_blocks_workspace(shape, bq, bk), "cuda")
    sa.mask_from_blocks(blocks, shape, bq, bk, True, ws, mb.struct)
    assert sa.read_status(mb.status) == sa.SA_OK
    valid = np.array([[not Pr.causal_future(qb, kb, N, bq, bk) for kb in range(nkb)] for qb in range(nqb)])
    want = m & valid
    got = mb.block_mask.cpu().numpy().reshape(B, Hq, nqb, nkb).astype(bool)
    assert np.array_equal(got, want)
    c = Pr.mask_to_csr(want)
    assert np.array_equal(mb.row_ptr.cpu().numpy(), c["row_ptr"])
    assert np.array_equal(mb.col_idx.cpu().numpy()[:c["kept_total"]], c["col_idx"])
    assert np.array_equal(mb.order.cpu().numpy(), c["order"])


def _fused_vs_separate(w, perm_np, q_bits, k_bits):
    """sa_reorder_predict_mask on original-order inputs against the oracle's
    reorder (bit-exact copies) and sa_predict_mask on those copies (same
    pooled values, mask, lists and order)."""
    import torch
    from long_context_mean_b200 import sa
    q_dev, k_dev = P.bf16_dev(q_bits), P.bf16_dev(k_bits)
    qr_want, kr_want = Y.reorder(q_bits, perm_np), Y.reorder(k_bits, perm_np)
    prm = sa.make_params(w.bq, w.bk, w.tau, w.theta, w.sink_tokens, w.txt_len, w.local_window,
                         w.anchor_tokens, w.causal)
    shape = sa.Shape(q_dev.shape[0], q_dev.shape[1], k_dev.shape[1], q_dev.shape[2], q_dev.shape[3],
                     q_dev.shape[3], sa.SA_BF16, 0)
    perm = torch.from_numpy(perm_np.astype(np.int32)).to("cuda")
    q_r = torch.full_like(q_dev, float("nan"))
    k_r = torch.full_like(k_dev, float("nan"))
    ws = sa.workspace(sa.predict_mask_workspace(shape, prm), "cuda")
    ws.fill_(0xFF)
    mb = sa.MaskBuffers.allocate(shape.B, shape.Hq, shape.N, prm.bq, prm.bk, "cuda")
    sa.reorder_predict_mask(perm, q_dev, k_dev, q_r, k_r, shape, prm, ws, mb.struct)
    assert sa.read_status(mb.status) == sa.SA_OK
    assert np.array_equal(q_r.cpu().view(torch.int16).numpy().view(np.uint16), qr_want)
    assert np.array_equal(k_r.cpu().view(torch.int16).numpy().view(np.uint16), kr_want)
    ref = run_gpu_predict(P.bf16_dev(qr_want), P.bf16_dev(kr_want), w, prm)
    off = sa.predict_mask_ws_layout(shape, prm)
    for i, key in ((0, "qhat"), (1, "khat"), (2, "s_q"), (3, "s_k")):
        if key == "khat":
            got = khat_from_ws(ws, off, shape.B, shape.Hkv, mb.struct.nkb, shape.d)
        else:
            n = ref[key].size
            got = ws[off[i]:off[i] + n * 4].view(torch.float32).cpu().numpy().reshape(ref[key].shape)
        assert np.array_equal(got, ref[key]), key
    assert np.array_equal(mb.block_mask.cpu().numpy().reshape(ref["mask"].shape).astype(bool), ref["mask"])
    kt = int(mb.kept_total.item())
    assert kt == ref["kept_total"]
    assert np.array_equal(mb.row_ptr.cpu().numpy(), ref["row_ptr"])
    assert np.array_equal(mb.col_idx.cpu().numpy()[:kt], ref["col_idx"][:kt])
    assert np.array_equal(mb.order.cpu().numpy(), ref["order"])


def test_reorder_predict_fused_small_window():
    w = I.Workload("fused_small", 321, 1, 3, 3, 5, 12, 20, 37, 128, 128, "bf16", "field", order="window",
                   win=(2, 8, 8), sink_frames=1, bq=128, bk=64, tau=0.5, theta=0.3, sigma=(1.0, 2.0, 2.0))
    g = I.gen_qkv(w)
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    _fused_vs_separate(w, np.asarray(perm), g["q_bits"], g["k_bits"])


def test_reorder_predict_fused_full_size_video():
    w = I.WORKLOADS["video"]
    g = I.gen_qkv(w)
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    _fused_vs_separate(w, np.asarray(perm), g["q_bits"], g["k_bits"])


def test_reorder_predict_rejects_out_of_range_perm():
    import torch
    from long_context_mean_b200 import sa
    N = 300
    shape = sa.Shape(1, 2, 2, N, 128, 128, sa.SA_BF16, 0)
    prm = sa.make_params(128, 64, 0.5)
    q = torch.randn(1, 2, N, 128, device="cuda").to(torch.bfloat16)
    k = torch.randn(1, 2, N, 128, device="cuda").to(torch.bfloat16)
    perm = torch.arange(N, dtype=torch.int32, device="cuda")
    perm[17] = N + 5                     # not a permutation: the kernel skips the token
    q_r, k_r = torch.empty_like(q), torch.empty_like(k)
    ws = sa.workspace(sa.predict_mask_workspace(shape, prm), "cuda")
    mb = sa.MaskBuffers.allocate(1, 2, N, 128, 64, "cuda")
    sa.reorder_predict_mask(perm, q, k, q_r, k_r, shape, prm, ws, mb.struct)
    assert sa.read_status(mb.status) == sa.SA_ERR_INVALID_ARG
