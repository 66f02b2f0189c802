"""Benchmark of the block-sparse attention forward path on B200.

One step = the whole path over one batch of synthetic input already resident
in HBM: layout build, reorder of Q, K, V, mask prediction (pooling, similarity
guard, compressed softmax + TopCdf, forced blocks, CSR lists, work order),
block-sparse attention with the PV skip, inverse reorder of O and LSE.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload video]
                    [--impl ours|reference]

Default workload: the video DiT attention (B=1, 24 heads, latent [13,30,52]
+ 226 text tokens, N = 20,506, d = 128, bf16, [2,8,8] windows, first-frame
sink, text forced, bq = 128, bk = 64, block sparsity 0.80, lambda = -5).

The metric is kept-block TFLOP/s: 4*d*(valid query x key pairs of the kept
tiles), the PV half counted only for tiles whose PV product ran, divided by
the device time of one step (CUDA events, L2 flushed between steps).  N > 1
ranks (torchrun) run independent replicas (the path has no exchange step);
value = all ranks' FLOPs / the slowest rank's time.

--impl reference times the fp64 CPU oracle (the plain restatement of the
method that the tests check the kernels against) on the same workload, one
bounded sample of query blocks per step, on this host's cores.
"""

from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse attn fwd ms & TFLOP/s (kept blocks) vs dense, N=20.5K video, 1×B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per launch of the attention kernel from the recorded ncu
# capture, keyed by the sha1 of the kernel code it was taken on (src_sha1);
# any other code reports null.
TRAFFIC = {("99b71bcd25c3ca8bef994bca62427ca1c63d45fe", "video"): 1.2109e9}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_sha1(name):
    """sha1 of a kernel source's code: comments and blank lines removed, so
    that a comment edit does not orphan the traffic measured for the code."""
    with open(os.path.join(ROOT, "long_context_mean_b200", "csrc", name)) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
    return hashlib.sha1("\n".join(lines).encode()).hexdigest()


# ----------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# FLOP accounting (algorithmic, from the mask lists and the PV-skip log)
# ----------------------------------------------------------------------------

def kept_flops(w, row_ptr, col_idx, skip, nqb):
    """4 * d * pairs split in QK (all kept tiles) and PV (unskipped tiles),
    pairs = valid query rows x valid (causally visible) keys of each tile."""
    import numpy as np
    N, bq, bk = w.N, w.bq, w.bk
    R = len(row_ptr) - 1
    qb = np.arange(R) % nqb
    counts = np.diff(row_ptr)
    rows = np.repeat(np.minimum(bq, N - qb * bq), counts)
    qbs = np.repeat(qb, counts)
    kb = col_idx[:row_ptr[-1]].astype(np.int64)
    cols = np.minimum(bk, N - kb * bk)
    if w.causal:
        i0 = qbs * bq
        pairs = np.zeros_like(kb)
        for r in range(bq):                      # rows of the block, vectorised over tiles
            i = i0 + r
            ok = i < N
            vis = np.clip(i - kb * bk + 1, 0, cols)
            pairs += np.where(ok, vis, 0)
    else:
        pairs = rows * cols
    qk = 2.0 * w.d * float(pairs.sum())
    pv = 2.0 * w.dv * float(pairs[skip[:row_ptr[-1]] == 0].sum())
    return qk, pv


def dense_flops(w):
    """Dense-equivalent op count of the attention: 2*(d + dv) per visible
    query-key pair over every head ([P3] 3.2: the "Speed" of a sparse kernel
    is this count divided by its latency, prediction included)."""
    pairs = w.N * (w.N + 1) / 2 if w.causal else float(w.N) * w.N
    return w.B * w.Hq * 2.0 * (w.d + w.dv) * pairs


def combined_sparsity(valid_tiles, kept, pv_skipped):
    """SpargeAttn's sparsity over both products ([P3] Table 6): skipped
    QK^T tiles plus skipped PV tiles over twice the valid tiles."""
    return (2.0 * (valid_tiles - kept) + pv_skipped) / (2.0 * valid_tiles)


def valid_tile_count(w, nqb, nkb):
    """Causally valid (query block, key block) tiles over batch and heads."""
    if w.causal:
        return w.B * w.Hq * sum(min(nkb, (min(w.N, (qb + 1) * w.bq) - 1) // w.bk + 1) for qb in range(nqb))
    return w.B * w.Hq * nqb * nkb


def spread(xs):
    """Median, p10 and p90 of a list of times (ms)."""
    import numpy as np
    a = np.asarray(xs, dtype=np.float64)
    return {"median": round(float(np.median(a)), 4), "p10": round(float(np.percentile(a, 10)), 4),
            "p90": round(float(np.percentile(a, 90)), 4), "mean": round(float(a.mean()), 4), "n": int(a.size)}


# ----------------------------------------------------------------------------
# Our arm
# ----------------------------------------------------------------------------

def workload_config(w, world):
    """The bench line's config: the workload with its sizes (both arms)."""
    return {"workload": f"{w.name}: B={w.B} H={w.Hq} N={w.N} ([{w.T},{w.H},{w.W}]+{w.txt_len} text) "
                        f"d={w.d} {w.order}{list(w.win) if w.order == 'window' else ''} sink_frames={w.sink_frames} "
                        f"bq={w.bq} bk={w.bk} tau={w.tau} theta={w.theta} lambda={w.lam}",
            "global_batch": w.B * world, "seq_len": w.N, "parallelism": f"replicas x{world}",
            "l2": "flushed between timed steps (256 MB write)"}


def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank timings (ms) over all ranks."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_tflops(world, flops_per_rank, ms):
    """Whole-job throughput: every replica processes flops_per_rank in the
    slowest rank's ms."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from long_context_mean_b200 import inputs as I
    from long_context_mean_b200 import sa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = I.WORKLOADS[args.workload]
    g = I.gen_qkv(w)
    host = {n: torch.from_numpy(g[n + "_bits"].view(np.int16)).view(torch.bfloat16).pin_memory() for n in "qkv"}
    q, k, v = (host[n].to(dev) for n in "qkv")
    # The step runs on a high-priority stream: the V reorder on the pipeline's
    # (default-priority) side stream then takes the SM slots the prediction
    # leaves free instead of competing with its HBM-bound pooling.
    stream = torch.cuda.Stream(device=dev, priority=torch.cuda.Stream.priority_range()[1])
    torch.cuda.set_stream(stream)
    pipe = sa.pipeline_for(w, device=dev, log_skips=True, qk8=args.qk8, order_group=args.order_group)

    # Calibration pass (untimed): mask, skip log, FLOPs, sparsity.
    pipe.run(q, k, v)
    st = pipe.status()
    if st != sa.SA_OK:
        raise RuntimeError(f"device status {sa.STATUS_NAMES.get(st, st)}")
    rp = pipe.mask.row_ptr.cpu().numpy().astype(np.int64)
    ci = pipe.mask.col_idx.cpu().numpy()
    skip = pipe.skip_log.cpu().numpy()
    nqb, nkb = pipe.mask.struct.nqb, pipe.mask.struct.nkb
    qk_flops, pv_flops = kept_flops(w, rp, ci, skip, nqb)
    flops = qk_flops + pv_flops
    kept = int(rp[-1])
    valid_tiles = valid_tile_count(w, nqb, nkb)
    sparsity = 1.0 - kept / valid_tiles
    pv_skipped = int(skip[:kept].sum())
    pipe.skip_log = None                      # timed steps run without the log

    # L2 flush buffer (larger than the 126 MB L2).
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def l2_flush():
        flush.fill_(1.0)

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def pred_stage(st):
        """Layout, reorders and mask prediction (the calls of Pipeline.run) on st."""
        if not pipe.identity:
            sa.layout_build(pipe.layout, pipe.perm, pipe.inv, pipe.layout_ws, st)
            # the V reorder on the pipeline's side stream, beside the prediction
            pipe.ev_layout.record(st)
            pipe.side.wait_event(pipe.ev_layout)
            sa.reorder(pipe.perm, v, pipe.vr, pipe.side)
            pipe.ev_v.record(pipe.side)
            # mask prediction with the reorder of Q and K fused into its pooling
            # pass (the 8-bit path: reorder and quantisation)
            if args.qk8:
                sa.reorder_predict_mask_q8(pipe.perm, q, k, args.qk8, pipe.q8, pipe.q_scales, pipe.k8,
                                           pipe.k_scales, pipe.shape, pipe.params, pipe.ws, pipe.mask.struct, st)
            else:
                sa.reorder_predict_mask(pipe.perm, q, k, pipe.qr, pipe.kr, pipe.shape, pipe.params, pipe.ws,
                                        pipe.mask.struct, st)
            st.wait_event(pipe.ev_v)
        else:
            if args.qk8:
                sa.reorder_predict_mask_q8(None, q, k, args.qk8, pipe.q8, pipe.q_scales, pipe.k8, pipe.k_scales,
                                           pipe.shape, pipe.params, pipe.ws, pipe.mask.struct, st)
            else:
                sa.predict_mask(q, k, pipe.shape, pipe.params, pipe.ws, pipe.mask.struct, st)

    def attn_stage(st):
        """Attention with the inverse reorder of O and LSE fused into its store."""
        if pipe.identity:
            qr, kr, vr = q, k, v
        else:
            qr, kr, vr = (q, k, pipe.vr) if args.qk8 else (pipe.qr, pipe.kr, pipe.vr)
        if args.qk8:
            sa.block_sparse_attn_qk8(pipe.q8, pipe.q_scales, pipe.k8, pipe.k_scales, vr, pipe.shape,
                                     pipe.mask.struct, pipe.lam, pipe.scale, pipe.out, pipe.attn_ws, pipe.lse,
                                     stream=st, out_perm=None if pipe.identity else pipe.perm, fmt=args.qk8)
        else:
            sa.block_sparse_attn(qr, kr, vr, pipe.shape, pipe.mask.struct, pipe.lam, pipe.scale, pipe.out,
                                 pipe.lse, stream=st, ws=pipe.attn_ws, out_perm=None if pipe.identity else pipe.perm)

    # The two stages as CUDA graphs (the inputs and buffers are fixed): a
    # replay launches every kernel of the stage without host gaps between them.
    graphs = None
    if not args.no_graphs:
        pred_stage(stream)               # warm-up of the library's one-time setup outside capture
        attn_stage(stream)
        torch.cuda.synchronize(dev)
        graphs = (torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph())
        cap = torch.cuda.Stream(device=dev, priority=stream.priority)
        with torch.cuda.graph(graphs[0], stream=cap, capture_error_mode="relaxed"):
            pred_stage(torch.cuda.current_stream(dev))
        with torch.cuda.graph(graphs[1], stream=cap, capture_error_mode="relaxed"):
            attn_stage(torch.cuda.current_stream(dev))
        torch.cuda.synchronize(dev)

    def step_timed():
        """One step with events around the stages: [start, after predict, after attention]."""
        e = [ev() for _ in range(3)]
        e[0].record(stream)
        if graphs:
            graphs[0].replay()
        else:
            pred_stage(stream)
        e[1].record(stream)
        if graphs:
            graphs[1].replay()
        else:
            attn_stage(stream)
        e[2].record(stream)
        return e

    # layout (1, Hilbert 3) + reorder V; pooling of Q and K (one launch), score, row scan, column
    # fill, order; attention
    launches_per_step = (0 if pipe.identity else (1 if w.order != "hilbert" else 3) + 1) + 5 + 1
    if args.qk8:
        launches_per_step += 1            # the tile-scale kernel (codes come from the pooling pass)

    for _ in range(args.warmup):
        l2_flush()
        step_timed()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(dev.index if dev.index is not None else 0) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    recs = []
    wall0 = time.perf_counter()
    for _ in range(args.steps):
        l2_flush()
        recs.append(step_timed())
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clk = clocks.stop() if clocks else None
    step_ms = [r[0].elapsed_time(r[2]) for r in recs]
    attn_ms = [r[1].elapsed_time(r[2]) for r in recs]
    pre_ms = [r[0].elapsed_time(r[1]) for r in recs]
    total_ms = sum(step_ms)
    st = pipe.status()
    if st != sa.SA_OK:
        raise RuntimeError(f"device status after timing {sa.STATUS_NAMES.get(st, st)}")

    # Dense reference kernel at the same shape (the speedup's denominator).
    od = torch.empty_like(pipe.out)
    ld = torch.empty(w.B, w.Hq, w.N, dtype=torch.float32, device=dev)
    dst = torch.zeros(1, dtype=torch.int32, device=dev)
    qr, kr, vr = (pipe.qr, pipe.kr, pipe.vr) if not (pipe.identity or args.qk8) else (q, k, v)
    dense = []
    dense_ws = sa.workspace(sa.attn_workspace(), dev)
    for i in range(args.warmup + max(3, min(args.steps, 10))):
        l2_flush()
        a, b = ev(), ev()
        a.record(stream)
        sa.dense_attn(qr, kr, vr, pipe.shape, w.causal, 0.0, od, ld, dst, ws=dense_ws)
        b.record(stream)
        if i >= args.warmup:
            dense.append((a, b))
    torch.cuda.synchronize(dev)
    dense_ms = statistics.median(x[0].elapsed_time(x[1]) for x in dense)
    # Per-row dropped mass alpha = 1 - exp(LSE_sparse - LSE_dense) ([P1] 3.2),
    # every row; the dense LSE comes back to the original token order when the
    # dense kernel ran on the reordered tensors.
    ld_h = ld.cpu().numpy().astype(np.float64)
    if qr is not q:
        perm_h = pipe.perm.cpu().numpy()
        back = np.empty_like(ld_h)
        back[..., perm_h] = ld_h
        ld_h = back
    alpha = 1.0 - np.exp(pipe.lse.cpu().numpy()[..., 0].astype(np.float64) - ld_h)
    worst = [int(x) for x in np.unravel_index(int(np.argmax(alpha)), alpha.shape)]
    alpha_rep = {"mean": float(alpha.mean()), "max": float(alpha.max()), "min": float(alpha.min()),
                 "worst_b_h_row": worst, "rows": int(alpha.size)}

    # End to end through the C ABI with host buffers (sa_forward_host, one call
    # per pass): pinned H2D of Q, K, V, the whole path, D2H of O and LSE, cut
    # into head chunks so the copies of one chunk overlap the kernels of the others.
    out_host = torch.empty(pipe.out.shape, dtype=pipe.out.dtype).pin_memory()
    lse_host = torch.empty(pipe.lse.shape, dtype=pipe.lse.dtype).pin_memory()
    e2e_ms = float("nan")
    if not args.qk8:   # the host-buffer pass runs the bf16 path
        hp = sa.host_pipeline_for(w, device=dev, chunks=args.e2e_chunks, order_group=args.order_group)

        def e2e_step():
            hp.run(host["q"], host["k"], host["v"], out_host, lse_host, stream)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize(dev)
        e2e = []
        for _ in range(args.steps):
            l2_flush()
            a, b = ev(), ev()
            a.record(stream)
            e2e_step()
            b.record(stream)
            e2e.append((a, b))
        torch.cuda.synchronize(dev)
        if hp.status() != sa.SA_OK:
            raise RuntimeError("device status after the end-to-end passes")
        e2e_ms = sum(x[0].elapsed_time(x[1]) for x in e2e) / len(e2e)
    h2d = sum(host[n].numel() * host[n].element_size() for n in "qkv")
    d2h = out_host.numel() * out_host.element_size() + lse_host.numel() * lse_host.element_size()

    # Max over ranks.
    mean_ms, attn_mean, e2e_ms = max_over_ranks([total_ms / args.steps, statistics.mean(attn_ms), e2e_ms],
                                                world, dev)
    if rank != 0:
        return None

    pk, pk_src = peaks()
    peak_tf = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_src = f"{pk_src} bf16 dense (burst)"
    if args.qk8:
        # QK at the 8-bit rate (the nominal int8 or fp8 / bf16 ratio 2 on the
        # measured bf16 peak), PV at the bf16 rate: the peak of the mixed contraction.
        peak_tf = flops / (qk_flops / (2 * peak_tf) + pv_flops / peak_tf)
        peak_src = f"{pk_src} bf16 (burst) x nominal {args.qk8}/bf16 ratio 2 on the QK half"
    attn_tf = flops / (attn_mean * 1e-3) / 1e12
    sha = src_sha1("attn_tc.cu")
    traffic = None if args.qk8 else TRAFFIC.get((sha, args.workload))
    res = {
        "metric": METRIC,
        "value": round(job_tflops(world, flops, mean_ms), 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(mean_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": f"bf16, QK {args.qk8} per block" if args.qk8 else "bf16",
        "data": "synthetic (seeded smooth-field generator, bf16)",
        "config": dict(workload_config(w, world), order_group=int(pipe.params.order_group),
                       launch="cuda graph per stage" if graphs else "eager"),
        "stages_ms": {"layout_reorder_predict": round(statistics.mean(pre_ms), 4),
                      "attention_with_fused_unreorder": round(statistics.mean(attn_ms), 4)},
        "timing_ms": {"step": spread(step_ms), "attention": spread(attn_ms), "prediction": spread(pre_ms)},
        "attn_ms": round(attn_mean, 4),
        "attn_tflops": round(attn_tf, 2),
        "dense_ms": round(dense_ms, 4),
        "speedup_vs_dense": round(dense_ms / attn_mean, 3),
        "speedup_vs_dense_whole_step": round(dense_ms / mean_ms, 3),
        "block_sparsity": round(sparsity, 4),
        "combined_qk_pv_sparsity": round(combined_sparsity(valid_tiles, kept, pv_skipped), 4),
        "dropped_mass_alpha": alpha_rep,
        "speed_dense_equiv_tops": round(dense_flops(w) / (mean_ms * 1e-3) / 1e12, 2),
        "speed_note": "dense op count / step time incl. prediction ([P3] 3.2 Speed)",
        "kept_tiles": kept,
        "valid_tiles": valid_tiles,
        "pv_skipped_tiles": pv_skipped,
        "flops_per_step": {"qk": qk_flops, "pv": pv_flops},
        "roofline": {"bound": "tensor", "achieved": round(attn_tf, 2), "peak": round(peak_tf, 1),
                     "unit": "TFLOP/s", "frac": round(attn_tf / peak_tf, 4), "traffic": traffic,
                     "peak_source": peak_src,
                     "kernel": f"attn_tc_kernel<64, {args.qk8} QK>" if args.qk8 else "attn_tc_kernel<64>"},
        "e2e": None if args.qk8 else {
            "value": round(job_tflops(world, flops, e2e_ms), 3), "unit": "TFLOP/s",
            "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "chunks": args.e2e_chunks, "entry_point": "sa_forward_host"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "wall_s": round(wall, 3),
    }
    if args.qk8:
        res["qk"] = f"{args.qk8}, per-block scales (Q per query block, K per key block); P, V bf16"
    if world == 1 and not args.no_cpu_baseline and not args.qk8:
        res["cpu_baseline"] = cpu_baseline(w, g, seconds=args.cpu_seconds)
    return res


def run_svg(args, rank, world, local_rank):
    """--path svg: the per-head spatial / temporal path (long_context_mean_b200.svg)
    on the workload's video shape.  Heads are biased to a frame (two in three)
    or to a position (one in three); the profile (dense attention and both
    candidates, sampled-row MSE, argmin) runs once before timing and is timed
    on its own; a step is the run: Q, K, V into each head's order and the
    block-sparse attention with the per-head store back."""
    import numpy as np
    import torch

    from long_context_mean_b200 import inputs as I
    from long_context_mean_b200 import sa, svg

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = I.WORKLOADS[args.workload]
    if w.B != 1 or w.Hq != w.Hkv or w.causal:
        raise SystemExit("--path svg needs a video workload with B = 1 and Hq = Hkv")
    bias = ["position" if h % 3 == 0 else "frame" for h in range(w.Hq)]
    g = I.biased_video_heads(w.T, w.H, w.W, w.txt_len, bias, d=w.d, dv=w.dv, seed=w.seed)
    q, k, v = (torch.from_numpy(g[n + "_bits"].view(np.int16)).to(dev).view(torch.bfloat16) for n in "qkv")
    stream = torch.cuda.current_stream(dev)
    pipe = svg.svg_pipeline_for(w, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    pipe.profile(q, k, v)                                 # warm-up profile
    prof = []
    for _ in range(3):
        flush.fill_(1.0)
        a, b = ev(), ev()
        a.record(stream)
        choice, _ = pipe.profile(q, k, v)
        b.record(stream)
        prof.append((a, b))
    torch.cuda.synchronize(dev)
    profile_ms = statistics.median(x[0].elapsed_time(x[1]) for x in prof)
    rp = pipe.mask.row_ptr.cpu().numpy().astype(np.int64)
    ci = pipe.mask.col_idx.cpu().numpy()
    nqb, nkb = pipe.mask.struct.nqb, pipe.mask.struct.nkb
    qk_flops, pv_flops = kept_flops(w, rp, ci, np.zeros(ci.size, dtype=np.uint8), nqb)
    flops = qk_flops + pv_flops
    kept = int(rp[-1])
    sparsity = 1.0 - kept / (w.Hq * nqb * nkb)

    def step_timed():
        e = [ev() for _ in range(3)]
        e[0].record(stream)
        sa.reorder_heads(pipe.perms, q, pipe.qr)
        sa.reorder_heads(pipe.perms, k, pipe.kr)
        sa.reorder_heads(pipe.perms, v, pipe.vr)
        e[1].record(stream)
        sa.block_sparse_attn(pipe.qr, pipe.kr, pipe.vr, pipe.shape, pipe.mask.struct, pipe.lam, pipe.scale,
                             pipe.out, pipe.lse, None, sa.SA_FLAG_OUT_PERM_PER_HEAD, ws=pipe.attn_ws,
                             out_perm=pipe.perms)
        e[2].record(stream)
        return e

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step_timed()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev.index if dev.index is not None else 0) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    recs = []
    for _ in range(args.steps):
        flush.fill_(1.0)
        recs.append(step_timed())
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    if pipe.status() != sa.SA_OK:
        raise RuntimeError("device status after the timed steps")
    step_ms = statistics.mean(r[0].elapsed_time(r[2]) for r in recs)
    attn_ms = statistics.mean(r[1].elapsed_time(r[2]) for r in recs)
    reorder_ms = statistics.mean(r[0].elapsed_time(r[1]) for r in recs)
    # dense kernel at the same shape
    od = torch.empty_like(pipe.out)
    dst = torch.zeros(1, dtype=torch.int32, device=dev)
    dense = []
    for i in range(args.warmup + 5):
        flush.fill_(1.0)
        a, b = ev(), ev()
        a.record(stream)
        sa.dense_attn(q, k, v, pipe.shape, False, 0.0, od, None, dst, ws=pipe.attn_ws)
        b.record(stream)
        if i >= args.warmup:
            dense.append((a, b))
    torch.cuda.synchronize(dev)
    dense_ms = statistics.median(x[0].elapsed_time(x[1]) for x in dense)
    step_ms, attn_ms = max_over_ranks([step_ms, attn_ms], world, dev)
    if rank != 0:
        return None
    pk, pk_src = peaks()
    peak_tf = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    attn_tf = flops / (attn_ms * 1e-3) / 1e12
    n_temporal = sum(1 for c in choice if c == svg.TEMPORAL)
    return {
        "metric": "per-head spatial/temporal sparse attn fwd TFLOP/s (kept blocks), video shape, 1xB200",
        "path": "svg",
        "value": round(job_tflops(world, flops, step_ms), 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (heads biased to a frame or a position, bf16)",
        "config": {"workload": f"{w.name} shape: B=1 H={w.Hq} N={w.N} ([{w.T},{w.H},{w.W}]+{w.txt_len} text) "
                               f"d={w.d} bq={w.bq} bk={w.bk}, per-head spatial/temporal placement",
                   "global_batch": world, "seq_len": w.N, "parallelism": f"replicas x{world}",
                   "l2": "flushed between timed steps (256 MB write)"},
        "stages_ms": {"reorder_heads_qkv": round(reorder_ms, 4), "attention_with_per_head_store": round(attn_ms, 4)},
        "profile_ms": round(profile_ms, 4),
        "heads_temporal": n_temporal,
        "heads_spatial": len(choice) - n_temporal,
        "dense_ms": round(dense_ms, 4),
        "speedup_vs_dense_whole_step": round(dense_ms / step_ms, 3),
        "block_sparsity": round(sparsity, 4),
        "kept_tiles": kept,
        "roofline": {"bound": "tensor", "achieved": round(attn_tf, 2), "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": round(attn_tf / peak_tf, 4), "traffic": None,
                     "peak_source": f"{pk_src} bf16 dense (burst)", "kernel": "attn_tc_kernel<64>"},
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
    }


SWEEP_TARGETS = (0.5, 0.6, 0.7, 0.8, 0.9, 0.95)
SWEEP_WORKLOADS = ("image", "video", "video_large")


def run_sweep(args, rank, world, local_rank):
    """--sweep: attention throughput against block sparsity ([P3] Fig. 10
    and Table 11: kernel speed as sparsity rises).  For each workload shape
    the similarity guard is off (theta = 0; the smooth-field generator's
    blocks sit below theta = 0.6, which would force every block) and tau is
    bisected on the library's own mask prediction until the kept-tile count
    reaches each target block sparsity; targets below the forced blocks'
    floor (sink and text rows and columns) report the floor.  One JSON line
    per point: tau, theta, the achieved sparsity, attention time (median of
    L2-flushed launches), kept-tile TFLOP/s, roofline fraction, dense time and
    speedup beside the ideal 1 / (1 - s)."""
    import numpy as np
    import torch

    from long_context_mean_b200 import inputs as I
    from long_context_mean_b200 import sa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    pk, pk_src = peaks()
    peak_tf = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    names = args.sweep.split(",") if args.sweep != "all" else list(SWEEP_WORKLOADS)
    lines = []
    for name in names:
        w = I.WORKLOADS[name].with_(theta=0.0)
        g = I.gen_qkv(w)
        q, k, v = (torch.from_numpy(g[n + "_bits"].view(np.int16)).to(dev).view(torch.bfloat16) for n in "qkv")
        del g
        pipe = sa.pipeline_for(w, device=dev, log_skips=True)
        pipe.run(q, k, v)
        if pipe.status() != sa.SA_OK:
            raise RuntimeError(f"{name}: device status {pipe.status()}")
        qr, kr, vr = (q, k, v) if pipe.identity else (pipe.qr, pipe.kr, pipe.vr)
        nqb, nkb = pipe.mask.struct.nqb, pipe.mask.struct.nkb
        valid = valid_tile_count(w, nqb, nkb)

        def timed(fn, n):
            ts = []
            for i in range(args.warmup + n):
                flush.fill_(1.0)
                a, b = ev(), ev()
                a.record(stream)
                fn()
                b.record(stream)
                if i >= args.warmup:
                    ts.append((a, b))
            torch.cuda.synchronize(dev)
            return [x[0].elapsed_time(x[1]) for x in ts]

        od = torch.empty_like(pipe.out)
        dst = torch.zeros(1, dtype=torch.int32, device=dev)
        dense_ms = statistics.median(timed(lambda: sa.dense_attn(qr, kr, vr, pipe.shape, w.causal, 0.0, od, None,
                                                                 dst, ws=pipe.attn_ws), 5))

        def predict(tau):
            pipe.params.tau = float(tau)
            if pipe.identity:
                sa.predict_mask(q, k, pipe.shape, pipe.params, pipe.ws, pipe.mask.struct)
            else:
                sa.reorder_predict_mask(pipe.perm, q, k, pipe.qr, pipe.kr, pipe.shape, pipe.params, pipe.ws,
                                        pipe.mask.struct)
            if pipe.status() != sa.SA_OK:
                raise RuntimeError(f"{name}: device status {pipe.status()} at tau {tau}")
            return 1.0 - int(pipe.mask.kept_total.item()) / valid

        floor = predict(1e-9)              # tau -> 0: one TopCdf block per row plus the forced ones
        for target in SWEEP_TARGETS:
            lo, hi, tau = 0.0, 1.0, 0.5
            s = predict(tau)
            for _ in range(30):             # sparsity falls as tau grows
                if abs(s - target) <= 0.002:
                    break
                lo, hi = (tau, hi) if s > target else (lo, tau)
                tau = 0.5 * (lo + hi)
                s = predict(tau)
            if target > floor:
                tau, s = 1e-9, predict(1e-9)
            skip = torch.zeros(pipe.mask.col_idx.numel(), dtype=torch.uint8, device=dev)
            sa.block_sparse_attn(qr, kr, vr, pipe.shape, pipe.mask.struct, w.lam, 0.0, pipe.out, pipe.lse, skip,
                                 ws=pipe.attn_ws, out_perm=None if pipe.identity else pipe.perm)
            rp = pipe.mask.row_ptr.cpu().numpy().astype(np.int64)
            ci = pipe.mask.col_idx.cpu().numpy()
            sk = skip.cpu().numpy()
            qk, pv = kept_flops(w, rp, ci, sk, nqb)
            kept = int(rp[-1])
            ms = timed(lambda: sa.block_sparse_attn(qr, kr, vr, pipe.shape, pipe.mask.struct, w.lam, 0.0, pipe.out,
                                                    pipe.lse, ws=pipe.attn_ws,
                                                    out_perm=None if pipe.identity else pipe.perm), 10)
            if pipe.status() != sa.SA_OK:
                raise RuntimeError(f"{name}: device status after the sweep point")
            att = statistics.median(ms)
            tf = (qk + pv) / (att * 1e-3) / 1e12
            line = {"sweep": name, "target_sparsity": target, "tau": round(tau, 6), "theta": 0.0, "lambda": w.lam,
                    "block_sparsity": round(s, 4), "forced_floor_sparsity": round(floor, 4),
                    "reached": abs(s - target) <= 0.005,
                    "combined_qk_pv_sparsity": round(combined_sparsity(valid, kept, int(sk[:kept].sum())), 4),
                    "kept_tiles": kept, "pv_skipped_tiles": int(sk[:kept].sum()),
                    "attn_ms": spread(ms), "attn_tflops": round(tf, 2),
                    "roofline_frac": round(tf / peak_tf, 4), "peak": peak_tf, "peak_source": f"{pk_src} bf16 (burst)",
                    "dense_ms": round(dense_ms, 4), "speedup_vs_dense": round(dense_ms / att, 3),
                    "ideal_speedup": round(1.0 / max(1e-9, 1.0 - s), 3),
                    "speed_dense_equiv_tops": round(dense_flops(w) / (att * 1e-3) / 1e12, 2)}
            lines.append(line)
            if rank == 0:
                print(json.dumps(line), flush=True)
        del pipe, q, k, v, qr, kr, vr
        torch.cuda.empty_cache()
    return None


# ----------------------------------------------------------------------------
# The oracle on the host cores (CPU baseline and the reference arm)
# ----------------------------------------------------------------------------

def oracle_sample_setup(w, g, head=0):
    """Oracle layout + mask for query head `head` of the first batch entry and
    the kv head it reads (one predict pass, fp64)."""
    from oracle import layout as Y
    from oracle import predict as Pr
    hk = head // (w.Hq // w.Hkv)
    perm, _ = Y.build_layout(w.order, w.T, w.H, w.W, w.win, w.sink_frames, w.txt_len)
    q = Y.reorder(g["q"][:1, head:head + 1], perm)
    k = Y.reorder(g["k"][:1, hk:hk + 1], perm)
    v = Y.reorder(g["v"][:1, hk:hk + 1], perm)
    r = Pr.predict_mask(q, k, w.bq, w.bk, w.tau, w.theta, w.causal, w.sink_tokens, w.txt_len,
                        w.local_window, w.anchor_tokens)
    return q, k, v, r["mask"]


def oracle_step(w, qkvm, qblocks):
    """The oracle's block-sparse attention on the given q-blocks of head 0;
    returns its kept-block FLOPs (QK + unskipped PV)."""
    from oracle import attention as A
    q, k, v, m = qkvm
    res = A.block_sparse_attention(q[0, 0], k[0, 0], v[0, 0], m[0, 0], w.bq, w.bk, w.causal, w.lam,
                                   qblocks=qblocks)
    fl = 0.0
    for (qb, kb), sk in res["skips"].items():
        rows = min(w.bq, w.N - qb * w.bq)
        cols = min(w.bk, w.N - kb * w.bk)
        fl += 2.0 * w.d * rows * cols + (0.0 if sk else 2.0 * w.dv * rows * cols)
    return fl


def cores_used():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(w, g, seconds=15.0):
    """The oracle on a bounded sample of the workload: query blocks of query
    head 0 in random order, then of head 1, and so on, until `seconds` of
    timed work (each head's oracle mask prediction is set-up, not timed)."""
    import numpy as np
    nqb = -(-w.N // w.bq)
    heads = g["q"].shape[1]
    fl, blocks, dt, h = 0.0, 0, 0.0, 0
    while dt < seconds and h < heads:
        qkvm = oracle_sample_setup(w, g, h)
        for qb in np.random.default_rng(h).permutation(nqb):
            t0 = time.perf_counter()
            fl += oracle_step(w, qkvm, [int(qb)])
            dt += time.perf_counter() - t0
            blocks += 1
            if dt >= seconds:
                break
        h += 1
    which = "query head 0" if h == 1 else f"query heads 0-{h - 1}"
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores_used(), "kind": "oracle",
            "sample": f"fp64 oracle block-sparse attention of {blocks} random query blocks of {which} "
                      f"(each head's mask predicted by the oracle, untimed), {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from long_context_mean_b200 import inputs as I
    w = I.WORKLOADS[args.workload]
    g = I.gen_qkv(w, heads=[0], batches=[0])
    qkvm = oracle_sample_setup(w, g)
    nqb = -(-w.N // w.bq)
    per_step = max(1, args.ref_qblocks)
    for i in range(args.warmup):
        oracle_step(w, qkvm, [(i * 7) % nqb])
    fl, t0 = 0.0, time.perf_counter()
    for s in range(args.steps):
        fl += oracle_step(w, qkvm, [((s * per_step + j) * 13) % nqb for j in range(per_step)])
    dt = time.perf_counter() - t0
    value = fl / dt / 1e12
    sample = (f"fp64 oracle block-sparse attention, {per_step} query blocks of head 0 per step "
              f"(mask predicted by the oracle for that head)")
    return {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores_used(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="video")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--qk8", choices=["int8", "e4m3"], default=None,
                    help="the predicted-mask path with 8-bit QK (per-block quantised Q and K)")
    ap.add_argument("--path", default="sparge", choices=["sparge", "svg"],
                    help="sparge: the predicted-mask path (the headline); svg: per-head spatial/temporal masks")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-qblocks", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", default=None,
                    help="attention throughput against block sparsity: 'all' or a comma list of workloads "
                         "(one JSON line per point instead of the headline line)")
    ap.add_argument("--no-graphs", action="store_true",
                    help="launch each kernel from the host every step instead of replaying CUDA graphs")
    ap.add_argument("--order-group", type=int, default=None,
                    help="work-order grouping of the mask rows (sa_mask_params.order_group); "
                         "default: the library's choice for the shape")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="head chunks of the end-to-end pass (copies overlap the kernels)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime
            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local_rank))
        try:
            if args.sweep:
                res = run_sweep(args, rank, world, local_rank)
            else:
                res = (run_svg if args.path == "svg" else run_ours)(args, rank, world, local_rank)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
