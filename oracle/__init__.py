"""Plain fp64 CPU oracle for the training-free block-sparse attention forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or link
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, header, table or helper with the CUDA library, and it never reads a
value produced by the CUDA library except where a test hands it one of several
equally correct results to check (a block mask whose only differences sit on a
TopCdf or similarity boundary, a PV-skip decision whose gap sits on lambda).

Every routine is written from the definitions on the source pages, in float64,
without blocking, fusion or reordering beyond what those definitions state.
The pages are cited by title and section:

* [P1] "AIGC 基本功｜视频稀疏注意力的误差与布局" (jefxiong.cn), sections 3.1-3.4
  (restricted softmax, error identity, spatial/temporal masks, permutation
  equivariance) and section 4 (block-occupancy ledger, worked example).
* [P2] MindIE-SD documentation page "稀疏" (rf_v2 / RainFusion2.0: block
  representatives, [t,h,w] window reorder, first-frame sink; ada_bsa).
* [P3] "SpargeAttention：中文精读笔记" (arXiv 2502.18137v8 reading notes),
  section 2.1 (sparse FlashAttention online softmax, M_g), 2.2 (selective token
  compression, CosSim guard, TopCdf), 2.3 (PV skip with lambda), 2.5 (Hilbert
  permutation), 3.2 (speed and sparsity definitions).
* [P4] "44. Local Sliding and Sparse Attention" (datawhale llm-algo-leetcode),
  Steps 2 and 4 (local causal mask, block-pair mask, access ledger).
* [P5] "78. Attention Access Pattern Benchmark" (datawhale llm-algo-leetcode),
  Steps 2 and 4 (selective sparse = window + anchors, coverage ledger).

Modules: ``attention`` (restricted softmax, tile recurrence, PV skip),
``layout`` (identity, window and Hilbert orders), ``predict`` (pooling,
CosSim, TopCdf, forced blocks), ``ledger`` (pair and tile ledgers),
``calibrate`` ((tau, theta) then lambda under L1 bounds, [P3] 2.4), ``quant``
(per-block INT8 / FP8 E4M3 QK, [P3] 2.4), ``svg`` (per-head spatial /
temporal candidates and their sampled-row choice, [P1] 3.3-5),
``tune_tau`` (the script that froze the workloads' tau).

Parity status per function is stated in each module header.  The pages name
no Hilbert variant; ``oracle.layout`` pins Skilling's curve against an
independent two-dimensional construction and the three-dimensional defining
properties of a Hilbert curve.
"""

from . import attention, layout, predict, ledger, calibrate, quant, svg  # noqa: F401
