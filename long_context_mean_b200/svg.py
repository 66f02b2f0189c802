"""Per-head spatial / temporal sparse attention with online profiling: the
Sparse VideoGen comparison of [P1] ("AIGC 基本功｜视频稀疏注意力的误差与布局",
sections 3.3, 3.4, 4 and 5).

Each head runs one of two fixed candidates: spatial (the pairs of one frame,
frame-major order) or temporal (the pairs of one position across frames,
token-major order); text tokens pair with every token.  ``profile`` draws a
few query rows, computes dense attention and both candidates, and picks per
head the candidate with the smaller mean squared output error on those rows;
only the sampled rows are computed (``sa_rows_attn``), densely and under
each candidate.
``run`` then enqueues, on one stream: Q, K, V into every head's own order
(one ``sa_reorder_heads`` pass each), block-sparse attention over the tile
covers, and the store back into the original order fused into the
attention epilogue (one permutation per head).

Every step runs in the library's kernels; this module allocates buffers,
draws the sampled rows (a seeded host generator, passed in as data) and
takes the argmin over the per-head errors that the GPU computed.
Restrictions: Hq == Hkv (the orders are per head and K, V are reordered
with them); no causal masking (video attention).
"""

from __future__ import annotations

import math

from . import sa

SPATIAL, TEMPORAL = sa.SA_HEAD_SPATIAL, sa.SA_HEAD_TEMPORAL


class SvgPipeline:
    def __init__(self, B, H, T, Hg, Wg, txt_len, d, dv, dtype="bf16", *, bq=128, bk=64, lam=-math.inf,
                 scale=0.0, flags=0, nrows=32, seed=0, device="cuda"):
        import torch
        self.T, self.Hg, self.Wg, self.txt_len = T, Hg, Wg, txt_len
        N = T * Hg * Wg + txt_len
        tdt = torch.bfloat16 if dtype in ("bf16", sa.SA_BF16) else torch.float32
        self.shape = sa.Shape(B, H, H, N, d, dv, sa.SA_BF16 if tdt == torch.bfloat16 else sa.SA_FP32, 0)
        self.bq, self.bk, self.lam, self.scale, self.flags = bq, bk, lam, scale, flags
        self.device = torch.device(device)
        BH = B * H
        self.kinds = torch.zeros(BH, dtype=torch.int32, device=device)
        self.perms = torch.empty(BH, N, dtype=torch.int32, device=device)
        self.mask = sa.MaskBuffers.allocate(B, H, N, bq, bk, device)
        self.mfb_ws = sa.workspace(sa.mask_from_blocks_workspace(self.shape, bq, bk), device)
        self.attn_ws = sa.workspace(sa.attn_workspace(), device)
        self.qr = torch.empty(B, H, N, d, dtype=tdt, device=device)
        self.kr = torch.empty(B, H, N, d, dtype=tdt, device=device)
        self.vr = torch.empty(B, H, N, dv, dtype=tdt, device=device)
        self.out = torch.empty(B, H, N, dv, dtype=tdt, device=device)
        self.lse = torch.empty(B, H, N, 1, dtype=torch.float32, device=device)
        # Sampled query rows: uniform with replacement over [0, N), at most N of them.
        g = torch.Generator().manual_seed(seed)
        rows = torch.randint(0, N, (min(nrows, N),), generator=g, dtype=torch.int64)
        self.rows = rows.to(torch.int32).to(device)
        self.mse = torch.zeros(2, BH, dtype=torch.float64, device=device)
        self.choice = None

    def place(self, kinds, stream=None):
        """Set the per-head candidates (a sequence of SPATIAL / TEMPORAL, or
        an int32 device tensor) and build the orders and tile lists."""
        import torch
        with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream(self.device)):
            if torch.is_tensor(kinds):
                self.kinds.copy_(kinds.to(torch.int32))
            else:
                self.kinds.copy_(torch.tensor(list(kinds), dtype=torch.int32))
            self.mask.status.zero_()
        sa.head_placement(self.T, self.Hg, self.Wg, self.txt_len, self.kinds, self.bq, self.bk, self.perms,
                          self.mask.block_mask, self.mask.status, stream)
        sa.mask_from_blocks(self.mask.block_mask, self.shape, self.bq, self.bk, False, self.mfb_ws,
                            self.mask.struct, stream)

    def run(self, q, k, v, stream=None, out=None, lse=None):
        """Enqueue the per-head sparse attention of the placed candidates;
        q, k, v BNSD in the original order, out/lse in the original order."""
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        sa.reorder_heads(self.perms, q, self.qr, stream)
        sa.reorder_heads(self.perms, k, self.kr, stream)
        sa.reorder_heads(self.perms, v, self.vr, stream)
        sa.block_sparse_attn(self.qr, self.kr, self.vr, self.shape, self.mask.struct, self.lam, self.scale, out, lse,
                             None, self.flags | sa.SA_FLAG_OUT_PERM_PER_HEAD, stream, ws=self.attn_ws,
                             out_perm=self.perms)
        return out, lse

    def profile(self, q, k, v, stream=None):
        """Online profiling on the sampled rows: their dense attention and
        their attention under each candidate (every head on that candidate),
        the MSE of each against dense, argmin per head (ties to spatial).
        Places the choice and returns (choice list, mse [2, heads] on the
        host)."""
        import torch
        BH = self.kinds.numel()
        nr = self.rows.numel()
        dv = self.shape.dv
        dense = torch.empty(BH, nr, dv, dtype=torch.float32, device=self.device)
        cand = torch.empty_like(dense)
        every = torch.arange(nr, dtype=torch.int32, device=self.device)
        st = torch.zeros(1, dtype=torch.int32, device=self.device)
        sa.rows_attn(q, k, v, self.shape, self.rows, dense, None, bq=self.bq, bk=self.bk, scale=self.scale,
                     status=st, stream=stream)
        for c in (SPATIAL, TEMPORAL):
            with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream(self.device)):
                self.kinds.fill_(c)
            sa.head_placement(self.T, self.Hg, self.Wg, self.txt_len, self.kinds, self.bq, self.bk, self.perms,
                              self.mask.block_mask, st, stream)
            sa.rows_attn(q, k, v, self.shape, self.rows, cand, None, self.perms, self.mask.block_mask, self.bq,
                         self.bk, self.scale, st, stream)
            sa.rows_mse(dense, cand, every, self.mse[c], st, stream)
        if sa.read_status(st, stream) != sa.SA_OK:
            raise RuntimeError("device status raised during profiling")
        mse = self.mse.cpu()
        choice = [TEMPORAL if float(mse[TEMPORAL, h]) < float(mse[SPATIAL, h]) else SPATIAL for h in range(BH)]
        self.place(choice, stream)
        self.choice = choice
        return choice, mse

    def status(self, stream=None) -> int:
        return sa.read_status(self.mask.status, stream)


def svg_pipeline_for(w, device="cuda", **kw) -> SvgPipeline:
    """SvgPipeline for a video workload description from ``inputs.WORKLOADS``."""
    if w.Hq != w.Hkv:
        raise ValueError("the per-head placement needs one K/V head per query head")
    return SvgPipeline(w.B, w.Hq, w.T, w.H, w.W, w.txt_len, w.d, w.dv, w.dtype, bq=w.bq, bk=w.bk,
                       device=device, **kw)
