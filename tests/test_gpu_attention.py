"""GPU parity: block-sparse and dense attention kernels against the fp64
oracle's tile recurrence, on masks the oracle chooses (handed to the GPU
through sa_mask_from_blocks)."""

import math

import numpy as np
import pytest

from long_context_mean_b200 import inputs as I
from oracle import attention as A
from oracle import predict as Pr
from tests import _parity as P

pytestmark = pytest.mark.gpu


def random_mask(rng, B, Hq, N, bq, bk, causal, p):
    nqb, nkb = -(-N // bq), -(-N // bk)
    m = rng.random((B, Hq, nqb, nkb)) < p
    for qb in range(nqb):
        for kb in range(nkb):
            if causal and Pr.causal_future(qb, kb, N, bq, bk):
                m[:, :, qb, kb] = False
    m[..., 0] = True            # key block 0 keeps every row non-empty
    return m


def run_sparse(q, k, v, mask_np, bq, bk, causal, lam, flags, scale=0.0, log=True):
    import torch
    from long_context_mean_b200 import sa
    shape = sa.make_shape(q, k, v)
    B, Hq, N = q.shape[:3]
    mb = sa.MaskBuffers.allocate(B, Hq, N, bq, bk, "cuda")
    ws = sa.workspace(sa.mask_from_blocks_workspace(shape, bq, bk), "cuda")
    blocks = torch.from_numpy(mask_np.astype(np.uint8).ravel()).to("cuda")
    sa.mask_from_blocks(blocks, shape, bq, bk, causal, ws, mb.struct)
    out = torch.full((B, Hq, N, v.shape[3]), float("nan"), dtype=q.dtype, device="cuda")
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    skip = torch.full((mb.col_idx.numel(),), 7, dtype=torch.uint8, device="cuda") if log else None
    sa.block_sparse_attn(q, k, v, shape, mb.struct, lam, scale, out, lse, skip, flags)
    st = sa.read_status(mb.status)
    res = {"status": st, "out": out.float().cpu().numpy(), "lse": lse.cpu().numpy(),
           "row_ptr": mb.row_ptr.cpu().numpy(), "col_idx": mb.col_idx.cpu().numpy(),
           "nqb": mb.struct.nqb}
    if log:
        res["skip"] = skip.cpu().numpy()
    return res


CASES = [
    # name, B, Hq, Hkv, N, d, dtype, bq, bk, causal, lam, p, flags
    ("fp32_toy", 1, 1, 1, 64, 16, "fp32", 16, 16, False, -math.inf, 0.5, 1),
    ("fp32_ragged", 2, 2, 1, 203, 32, "fp32", 32, 16, True, -math.inf, 0.4, 1),
    ("bf16_simt_lam", 1, 3, 3, 700, 128, "bf16", 128, 64, False, -2.0, 0.5, 1),
    ("bf16_simt_causal_gqa", 1, 4, 2, 900, 128, "bf16", 128, 64, True, -3.0, 0.6, 1),
    ("bf16_simt_bk128", 1, 2, 2, 650, 128, "bf16", 128, 128, False, -math.inf, 0.5, 1),
    ("bf16_simt_d64", 2, 2, 2, 333, 64, "bf16", 64, 32, True, -1.0, 0.5, 1),
    # the same shapes on the default path (tensor cores where they apply)
    ("bf16_tc_lam", 1, 3, 3, 700, 128, "bf16", 128, 64, False, -2.0, 0.5, 0),
    ("bf16_tc_causal_gqa", 1, 4, 2, 900, 128, "bf16", 128, 64, True, -3.0, 0.6, 0),
    ("bf16_tc_bk128", 1, 2, 2, 650, 128, "bf16", 128, 128, False, -math.inf, 0.5, 0),
    ("bf16_tc_causal_bk128", 2, 2, 1, 1100, 128, "bf16", 128, 128, True, -math.inf, 0.7, 0),
    ("bf16_tc_dense_mask", 1, 2, 2, 1024, 128, "bf16", 128, 64, False, -math.inf, 1.0, 0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_block_sparse_vs_oracle(case):
    import torch
    name, B, Hq, Hkv, N, d, dt, bq, bk, causal, lam, p, flags = case
    rng = np.random.default_rng(len(name) * 31 + N)
    w = I.Workload(name, 500 + N, B, Hq, Hkv, 1, 1, N, 0, d, d, dt, "field" if Hq == Hkv else "lowrank",
                   sigma=(0.0, 0.0, 8.0), sigma_pos=30.0, noise=0.5)
    g = I.gen_qkv(w)
    q, k, v = P.qkv_dev(g, dt)
    m = random_mask(rng, B, Hq, N, bq, bk, causal, p)
    r = run_sparse(q, k, v, m, bq, bk, causal, lam, flags)
    assert r["status"] == 0
    ref = A.block_sparse_attention_heads(g["q"], g["k"], g["v"], m, bq, bk, causal, lam)
    if lam > -math.inf:
        over = P.skip_override_from_gpu(r["skip"], r["row_ptr"], r["col_idx"], r["nqb"], B, Hq)
        nb = P.check_skip_decisions(over, ref["skips"], ref["gaps"], lam)
        if nb:
            ref = A.block_sparse_attention_heads(g["q"], g["k"], g["v"], m, bq, bk, causal, lam,
                                                 skip_override=over, band=P.LAMBDA_BAND)
    else:
        assert not r["skip"][:int(r["row_ptr"][-1])].any()
    P.attention_check(r["out"], r["lse"], ref)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("flags", [0, 1])
def test_dense_vs_oracle(causal, flags):
    import torch
    from long_context_mean_b200 import sa
    B, Hq, Hkv, N, d = 1, 2, 2, 777, 128
    w = I.Workload("dense", 901, B, Hq, Hkv, 1, 1, N, 0, d, d, "bf16", "iid")
    g = I.gen_qkv(w)
    q, k, v = P.qkv_dev(g, "bf16")
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.dense_attn(q, k, v, sa.make_shape(q, k, v), causal, 0.0, out, lse, st, flags)
    assert sa.read_status(st) == 0
    for h in range(Hq):
        y, l = A.dense_attention(g["q"][0, h], g["k"][0, h], g["v"][0, h], causal)
        ref = {"out": y[None, None], "lse": l[None, None]}
        P.attention_check(out[:, h:h + 1].float().cpu().numpy(), lse[:, h:h + 1].cpu().numpy(), ref)


def test_two_key_counterexample_on_gpu():
    """q = [1], keys [ln 99, 0], values [0, 100]: full attention gives 1, the
    pruned mask (first key only) gives 0 (error-and-layout page, 3.2)."""
    import torch
    from long_context_mean_b200 import sa
    c = I.two_key_inputs()
    d = 4                      # pad to the smallest supported width with zeros
    q = np.zeros((1, 1, 2, d), np.float32)
    k = np.zeros((1, 1, 2, d), np.float32)
    v = np.zeros((1, 1, 2, d), np.float32)
    q[0, 0, :, 0] = 1.0
    k[0, 0, :, 0] = c["k"][:, 0]
    v[0, 0, :, 0] = c["v"][:, 0]
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
    full = np.ones((1, 1, 2, 2), bool)
    pruned = np.array([[[[True, False], [True, False]]]])
    r1 = run_sparse(qd, kd, vd, full, 1, 1, False, -math.inf, 1, scale=1.0)
    r0 = run_sparse(qd, kd, vd, pruned, 1, 1, False, -math.inf, 1, scale=1.0)
    assert r1["out"][0, 0, 0, 0] == pytest.approx(1.0, abs=1e-5)
    assert r0["out"][0, 0, 0, 0] == pytest.approx(0.0, abs=1e-6)


@pytest.mark.parametrize("flags", [0, 1])
@pytest.mark.parametrize("causal", [False, True])
def test_pv_skip_exercised(flags, causal):
    """Queries share one direction and the keys' weight on it falls along the
    sequence, so later key blocks sit far below the running max and the
    lambda test skips their PV product."""
    import torch
    B, Hq, N, d, bq, bk, lam = 1, 2, 1024, 128, 128, 64, -4.0
    rng = np.random.default_rng(42)
    u = rng.normal(size=d)
    u /= np.linalg.norm(u)
    q = (3.0 * u + 0.3 * rng.normal(size=(B, Hq, N, d))).astype(np.float32)
    k = (np.linspace(4, -4, N)[:, None] * u * 6.0 + 0.3 * rng.normal(size=(B, Hq, N, d))).astype(np.float32)
    v = rng.normal(size=(B, Hq, N, d)).astype(np.float32)
    bits = {n: I.to_bf16_bits(x) for n, x in (("q", q), ("k", k), ("v", v))}
    qf, kf, vf = (I.bf16_bits_to_f32(bits[n]) for n in "qkv")
    qd, kd, vd = (P.bf16_dev(bits[n]) for n in "qkv")
    m = random_mask(np.random.default_rng(1), B, Hq, N, bq, bk, causal, 0.8)
    r = run_sparse(qd, kd, vd, m, bq, bk, causal, lam, flags)
    assert r["status"] == 0
    ref = A.block_sparse_attention_heads(qf, kf, vf, m, bq, bk, causal, lam)
    over = P.skip_override_from_gpu(r["skip"], r["row_ptr"], r["col_idx"], r["nqb"], B, Hq)
    if P.check_skip_decisions(over, ref["skips"], ref["gaps"], lam):
        ref = A.block_sparse_attention_heads(qf, kf, vf, m, bq, bk, causal, lam, skip_override=over,
                                             band=P.LAMBDA_BAND)
    n_skip = sum(ref["skips"].values())
    assert n_skip >= 10, n_skip
    P.attention_check(r["out"], r["lse"], ref)


@pytest.mark.parametrize("path", ["tc", "simt", "int8", "e4m3"])
def test_undersized_mask_attention_stays_in_bounds(path):
    """A mask whose lists overflow col_capacity (the builder raises
    SA_ERR_CAPACITY), handed to attention on the same stream before the
    status is read: the attention kernels must not read or write past the
    capacity.  Canary bytes after the skip log's and the 8-bit path's
    tile-scale entries stay untouched, and the status word keeps
    SA_ERR_CAPACITY."""
    import torch
    from long_context_mean_b200 import sa
    N, bq, bk, cap = 512, 128, 64, 31          # 4 x 8 = 32 kept tiles, one over
    rng = np.random.default_rng(11)
    q, k, v = (P.bf16_dev(I.to_bf16_bits(rng.standard_normal((1, 1, N, 128)).astype(np.float32)))
               for _ in range(3))
    shape = sa.make_shape(q, k, v)
    mb = sa.MaskBuffers.allocate(1, 1, N, bq, bk, "cuda", capacity=cap)
    ws = sa.workspace(sa.mask_from_blocks_workspace(shape, bq, bk), "cuda")
    sa.mask_from_blocks(torch.ones(4 * 8, dtype=torch.uint8, device="cuda"), shape, bq, bk, False, ws, mb.struct)
    canary = 0xA5
    skip = torch.full((cap + 64,), canary, dtype=torch.uint8, device="cuda")
    out = torch.zeros((1, 1, N, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, N), dtype=torch.float32, device="cuda")
    if path in ("tc", "simt"):
        flags = sa.SA_FLAG_FORCE_SIMT if path == "simt" else 0
        sa.block_sparse_attn(q, k, v, shape, mb.struct, -1.0, 0.0, out, lse, skip, flags)
        aws = None
    else:
        q8 = torch.empty((1, 1, N, 128), dtype=torch.uint8, device="cuda")
        k8 = torch.empty_like(q8)
        qs = torch.empty(N // bq, dtype=torch.float32, device="cuda")
        ks = torch.empty(N // bk, dtype=torch.float32, device="cuda")
        sa.quantize_blocks(q, bq, q8, qs, path)
        sa.quantize_blocks(k, bk, k8, ks, path)
        need = sa.attn_qk8_workspace(mb.struct)
        aws = torch.full((need + 256,), canary, dtype=torch.uint8, device="cuda")
        sa.block_sparse_attn_qk8(q8, qs, k8, ks, v, shape, mb.struct, -1.0, 0.0, out, aws, lse, skip, fmt=path)
    assert sa.read_status(mb.status) == sa.SA_ERR_CAPACITY
    sk = skip.cpu().numpy()
    assert (sk[cap:] == canary).all(), "skip log written past col_capacity"
    rp = mb.row_ptr.cpu().numpy()
    assert rp[-1] == 32 and rp[3] == 24
    assert set(sk[:24].tolist()) <= {0, 1}, "rows inside the capacity must still be computed"
    if aws is not None:
        a = aws.cpu().numpy()
        assert (a[256 + 4 * cap:] == canary).all(), "tile scales written past col_capacity"
    # rows of query blocks 0-2 were computed; block 3 (list past capacity) was left alone
    o = out.float().cpu().numpy()[0, 0]
    assert np.isfinite(o[:3 * bq]).all() and (np.abs(o[:3 * bq]).sum(axis=1) > 0).all()
    assert (o[3 * bq:] == 0).all()


@pytest.mark.parametrize("bk", [64, 128])
def test_timeout_path_reports_and_recovers(bk):
    """The bounded waits' error path in the form this pool allows (no GPU
    fault, no endless wait): SA_FLAG_TEST_STALL makes the first CTA of the
    tensor-core kernel load no K tile, so its waits run out after 10 ms.  The
    call must report SA_ERR_TIMEOUT, every role must stop issuing and drain,
    the CTA must release its TMEM, and later calls on the same context must
    run normally and match the oracle (twice, so a leak of TMEM or of a
    barrier phase would show)."""
    from long_context_mean_b200 import sa
    N, bq = 2048, 128
    w = I.Workload("stall", 4321, 1, 4, 4, 1, 1, N, 0, 128, 128, "bf16", "field", sigma=(0.0, 0.0, 8.0), noise=0.5)
    g = I.gen_qkv(w)
    q, k, v = P.qkv_dev(g, "bf16")
    rng = np.random.default_rng(bk)
    m = random_mask(rng, 1, 4, N, bq, bk, False, 0.5)
    assert sa.attn_kernel_path(sa.make_shape(q, k, v), bq, bk) == 1
    for _ in range(2):
        r = run_sparse(q, k, v, m, bq, bk, False, -math.inf, sa.SA_FLAG_TEST_STALL, log=False)
        assert r["status"] == sa.SA_ERR_TIMEOUT
        r = run_sparse(q, k, v, m, bq, bk, False, -math.inf, 0, log=False)
        assert r["status"] == sa.SA_OK
        ref = A.block_sparse_attention_heads(g["q"], g["k"], g["v"], m, bq, bk, False)
        P.attention_check(r["out"], r["lse"], ref)
