"""GPU parity: token layouts and reorders, bit-exact against the oracle."""

import numpy as np
import pytest

from long_context_mean_b200 import inputs as I
from oracle import layout as Y

pytestmark = pytest.mark.gpu

CASES = [
    ("window", 13, 30, 52, 226, 1, (2, 8, 8)),     # the video workload
    ("hilbert", 21, 45, 80, 0, 1, (1, 1, 1)),      # the large video workload
    ("window", 5, 7, 9, 3, 0, (2, 3, 4)),          # edge windows on every axis
    ("window", 4, 4, 4, 0, 0, (4, 1, 1)),          # position-major (worked example)
    ("hilbert", 6, 5, 7, 3, 1, (1, 1, 1)),         # non-cubic box with sink and text
    ("hilbert", 1, 1, 1, 0, 0, (1, 1, 1)),         # a single token
    ("hilbert", 9, 16, 16, 0, 1, (1, 1, 1)),       # full 8x16x16 body
    ("identity", 3, 10, 10, 5, 0, (1, 1, 1)),
]


@pytest.mark.parametrize("mode,T,H,W,txt,sink,win", CASES)
def test_layout_bit_exact(mode, T, H, W, txt, sink, win):
    import torch
    from long_context_mean_b200 import sa
    n = T * H * W + txt
    desc = sa.make_layout(T, H, W, txt, sink, mode, win)
    perm = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    inv = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    ws = sa.workspace(sa.layout_workspace(desc), "cuda")
    sa.layout_build(desc, perm, inv, ws)
    ref_perm, ref_inv = Y.build_layout(mode, T, H, W, win, sink, txt)
    assert np.array_equal(perm.cpu().numpy(), ref_perm)
    assert np.array_equal(inv.cpu().numpy(), ref_inv)


@pytest.mark.parametrize("row,dtype", [(128, "bf16"), (16, "fp32"), (1, "fp32"), (64, "bf16"), (3, "bf16")])
def test_reorder_unreorder_bit_exact(row, dtype):
    import torch
    from long_context_mean_b200 import sa
    rng = np.random.default_rng(row)
    outer, N = 3, 1001
    perm_np = rng.permutation(N).astype(np.int32)
    x_np = rng.normal(size=(outer, N, row)).astype(np.float32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.from_numpy(x_np).to("cuda").to(tdt)
    perm = torch.from_numpy(perm_np).to("cuda")
    y = torch.empty_like(x)
    sa.reorder(perm, x, y)
    xb = x.float().cpu().numpy()
    assert np.array_equal(y.float().cpu().numpy(), Y.reorder(xb, perm_np, axis=1))
    z = torch.empty_like(x)
    sa.unreorder(perm, y, z)
    assert np.array_equal(z.float().cpu().numpy(), xb)


def test_reorder_video_qkv_shape():
    import torch
    from long_context_mean_b200 import sa
    w = I.WORKLOADS["video"]
    perm_np, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    x = torch.randn(1, 4, w.N, 128, device="cuda", dtype=torch.bfloat16)
    y = torch.empty_like(x)
    perm = torch.from_numpy(perm_np.astype(np.int32)).to("cuda")
    sa.reorder(perm, x, y)
    assert torch.equal(y, x[:, :, perm.long()])
