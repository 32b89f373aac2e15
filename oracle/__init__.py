"""Plain fp64 CPU oracle for ASA block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path; the one common module is the seeded input generator
(``block_sparse_attention_asa_b200.workloads``), which holds none of the
method's arithmetic.

What it computes, and from where:

* ``asa``       -- the content-aware block mask of BLADE's Adaptive Block-Sparse
                   Attention (BLADE digest, abstract and "方法详解 / 关键设计":
                   keep the blocks whose mutual relevance is high).  The pages do
                   not define the scoring; the reading used here is: mean-pool Q
                   and K per token block, softmax of pooled scores, keep by top-k
                   or smallest prefix reaching a cumulative mass, ties to the
                   lowest block index, optional cap and forced blocks.
* ``patterns``  -- the fixed masks M0-M4 of the Sparse-vDiT blog ("四种注意力模式"
                   table) and the 3D attention tile of the Efficient-vDiT blog
                   ("3.1 注意力图块化"), as exact token-level closed forms.
* ``attention`` -- softmax(Q Kᵀ/√d) V per head (Sparse-vDiT blog, "核心公式 /
                   全注意力机制") restricted to the kept blocks, with the
                   log-sum-exp; an empty row (skip head, M1) gives O = 0.
* ``backward``  -- dQ, dK, dV of the masked attention for a given dO (BLADE
                   digest, "技术框架": ASA is trained jointly, so the attention is
                   differentiated; the mask is a constant of the step), and the
                   transpose of a CSR block mask.
* ``search``    -- the offline pattern-search quantities of the Sparse-vDiT blog
                   ("离线搜索损失函数", "注意力模式选择", Algorithm 1): per-head
                   MSE against full attention, pattern sparsity, the loss
                   L_i = MSE + lambda (1 - S_i) and the eps selection rule.

Parity pins (``tests/test_oracle_*.py``): dense attention vs torch's float64
``scaled_dot_product_attention``; pooling vs ``avg_pool1d``; selection vs
brute-force subset enumeration; patterns vs token-pair enumeration; the
invariants of a convex combination; a hand-computable worked example; the
gradients vs torch float64 autograd of SDPA and vs central finite differences
of the forward oracle, with the softmax's shift and scaling identities.  The
3D-tile pattern is pinned by a hand derivation for frames that straddle
blocks (``tests/golden/tile3d_example.json``); the block reading it checks is
the plainest one the Efficient-vDiT page's section 3.1 allows.
"""
from .asa import pool, pooled_probs, select_row, asa_mask, MaskInfo  # noqa: F401
from .patterns import pattern_row, pattern_mask, keep_token_pair  # noqa: F401
from .attention import masked_attention, attention_rows, attention_probs  # noqa: F401
from .backward import attention_backward, attention_backward_sampled, mask_transpose  # noqa: F401
from . import search  # noqa: F401
