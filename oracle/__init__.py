"""fp64 CPU oracle for sparse + linear video attention -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously-correct numpy restatement of what the
three source write-ups define:

* ``oracle.sla``    -- SLA (Sparse-Linear Attention, arXiv 2509.24006), as
                       described on the techwalker page "清华大学破解视频生成
                       卡顿难题", section 3 ("SLA方法的核心机制"): block mean
                       pooling, the compressed score matrix P_c, the 5 % / 10 %
                       percentile classification, sparse softmax attention on
                       critical blocks, linear attention on marginal blocks and
                       the learnable projection of the linear output.
* ``oracle.sla_grad`` -- the SLA backward (same page, section 3, last paragraph):
                       FlashAttention-style gradients of the sparse part and
                       the gradients of the normalised linear part, the block
                       mask held fixed.
* ``oracle.lvsa``   -- LVSA (arXiv 2605.31057), as described on the rainbus
                       paper-digest page, sections "核心方法" and "方法步骤详情":
                       the global period T_per, the rotating global set G_s,
                       the adaptive and expanded local window, the attention set
                       A(t) and exact softmax over the attended frames.
* ``oracle.tile3d`` -- RoPeSLR (arXiv 2605.20659), as described on the
                       aixinbiao blog page, section "稀疏邻域加低秩远场": a
                       3x3x3 local neighbourhood, a pooled low-rank far field
                       and the gate g*local + (1-g)*global.
* ``oracle.sta``    -- the 3-D sliding tile attention mask of VORTA (arXiv
                       2505.18809), as described on the zhaoyang97 paper-notes
                       page, section "方法详解", design 1, and attention over it.
* ``oracle.svoo``   -- SVOO (arXiv 2603.18636), as described on the gist.science
                       summary, section 3, stage 2: bidirectional Q-K
                       co-clustering from sampled anchors, and attention over
                       the top block pairs of the co-clustered order.

It shares no code with the CUDA library and imports nothing from it.  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
use it; the product path never does.

All arithmetic is fp64.  Parity status of every function is listed in each
module's header; every function is pinned by a test in ``tests/test_oracle_*.py``
against closed forms, special cases, library routines or hand-worked examples.
"""
from . import sla, sla_grad, lvsa, tile3d, sta, svoo  # noqa: F401
