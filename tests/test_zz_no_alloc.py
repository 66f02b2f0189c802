"""sa_predict_mask_noalloc (scratch held by the library) gives the same mask,
lists and work order as sa_predict_mask with a caller workspace, call after
call.  Collected last so that it also runs after every other GPU test has
used the library in the same process."""

import ctypes

import numpy as np
import pytest

from long_context_mean_b200 import inputs as I
from oracle import layout as Y
from tests import _parity as P

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 32 << 20


def _shape_of(q_dev, k_dev):
    from long_context_mean_b200 import sa
    return sa.Shape(q_dev.shape[0], q_dev.shape[1], k_dev.shape[1], q_dev.shape[2], q_dev.shape[3],
                    q_dev.shape[3], sa.dtype_code(q_dev), 0)


def _predict(q_dev, k_dev, params, noalloc):
    from long_context_mean_b200 import sa
    shape = _shape_of(q_dev, k_dev)
    mb = sa.MaskBuffers.allocate(shape.B, shape.Hq, shape.N, params.bq, params.bk, "cuda")
    mb.block_mask.fill_(0xAB)
    mb.row_ptr.fill_(-7)
    mb.col_idx.fill_(-7)
    mb.order.fill_(-7)
    if noalloc:
        sa.predict_mask_noalloc(q_dev, k_dev, shape, params, mb.struct)
    else:
        ws = sa.workspace(sa.predict_mask_workspace(shape, params), "cuda")
        ws.fill_(0xFF)
        sa.predict_mask(q_dev, k_dev, shape, params, ws, mb.struct)
    status = sa.read_status(mb.status)
    kt = int(mb.kept_total.item())
    return {
        "status": status,
        "kept_total": kt,
        "mask": mb.block_mask.cpu().numpy(),
        "row_ptr": mb.row_ptr.cpu().numpy(),
        "col_idx": mb.col_idx[:kt].cpu().numpy(),
        "order": mb.order.cpu().numpy(),
    }


def _assert_same(a, b):
    assert a["status"] == b["status"] == 0
    assert a["kept_total"] == b["kept_total"] > 0
    for key in ("mask", "row_ptr", "col_idx", "order"):
        assert np.array_equal(a[key], b[key]), key


def _video_case():
    """The video DiT workload (13x30x52 latent grid + 226 text tokens, 24
    heads, d = 128, bf16) in its [2,8,8]-window order."""
    from long_context_mean_b200 import sa
    w = I.WORKLOADS["video"]
    g = I.gen_qkv(w)
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    q_dev = P.bf16_dev(Y.reorder(g["q_bits"], perm))
    k_dev = P.bf16_dev(Y.reorder(g["k_bits"], perm))
    prm = sa.make_params(w.bq, w.bk, w.tau, w.theta, w.sink_tokens, w.txt_len, w.local_window,
                         w.anchor_tokens, w.causal)
    return q_dev, k_dev, prm


def _guard_case():
    """Two batches, similarity guard on, ragged last blocks."""
    from long_context_mean_b200 import sa
    w = I.Workload("noalloc_guard", 4242, 2, 3, 3, 1, 1, 513, 0, 128, 128, "bf16", "field",
                   bq=128, bk=64, tau=0.5, theta=0.25, sigma=(0.0, 0.0, 6.0), sigma_pos=20.0)
    g = I.gen_qkv(w)
    q_dev, k_dev, _ = P.qkv_dev(g, "bf16")
    return q_dev, k_dev, sa.make_params(128, 64, 0.5, 0.25)


def test_two_calls_in_a_row_match_workspace_entry_point():
    video = _video_case()
    guard = _guard_case()
    ref_video = _predict(*video, noalloc=False)
    ref_guard = _predict(*guard, noalloc=False)
    # Two calls in a row on different problems, then the first problem again
    # (the scratch holds the previous call's values when each call starts).
    _assert_same(_predict(*video, noalloc=True), ref_video)
    _assert_same(_predict(*guard, noalloc=True), ref_guard)
    _assert_same(_predict(*video, noalloc=True), ref_video)


def test_largest_shipped_shape_fits():
    """32 query heads over 8 kv heads of 131,072 causal tokens (the long
    causal LM workload's shape) stays inside the fixed scratch."""
    import torch
    from long_context_mean_b200 import sa
    w = I.WORKLOADS["lm_causal"]
    gen = torch.Generator(device="cuda").manual_seed(5)
    q_dev = torch.randn(1, w.Hq, w.N, w.d, device="cuda", generator=gen).to(torch.bfloat16)
    k_dev = torch.randn(1, w.Hkv, w.N, w.d, device="cuda", generator=gen).to(torch.bfloat16)
    prm = sa.make_params(w.bq, w.bk, w.tau, w.theta, 0, 0, w.local_window, w.anchor_tokens, w.causal)
    assert sa.predict_mask_workspace(_shape_of(q_dev, k_dev), prm) <= SCRATCH_LIMIT
    ref = _predict(q_dev, k_dev, prm, noalloc=False)
    _assert_same(_predict(q_dev, k_dev, prm, noalloc=True), ref)
    _assert_same(_predict(q_dev, k_dev, prm, noalloc=True), ref)


def test_oversized_shape_is_rejected_before_any_work():
    from long_context_mean_b200 import sa
    lib = sa.load()
    shape = sa.Shape(1, 64, 8, 200000, 128, 128, sa.SA_BF16, 0)
    prm = sa.make_params(128, 64, 0.9)
    assert sa.predict_mask_workspace(shape, prm) > SCRATCH_LIMIT
    fake = ctypes.c_void_p(4096)   # never dereferenced: the size check comes first
    m = sa.Mask(4096, 4096, 4096, 4096, 4096, 4096, 100, 0, 0, 0, 0, 0, 0)
    rc = lib.sa_predict_mask_noalloc(fake, fake, ctypes.byref(shape), ctypes.byref(prm), ctypes.byref(m),
                                     ctypes.c_void_p(None))
    assert rc == sa.SA_ERR_WORKSPACE
    assert b"sa_predict_mask_noalloc" in lib.sa_last_error()
