"""fp64 CPU oracle for exact scaled-dot-product attention (test infrastructure).

This package is test infrastructure, not part of the product. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline legs of ``bench.py`` may import
it. It shares no code with the CUDA library and imports nothing from it.

Sources, named by page and section (all four pages describe FlashAttention,
Dao et al., NeurIPS 2022):
  [card]      "FlashAttention" concept card (lukebest.github.io/concepts/flashattention):
              sections "算法要点" (online softmax, recompute in backward, kernel
              fusion with mask), "Block-Sparse FlashAttention", "IO 复杂度".
  [interview] FlashAttention interview explainer (mstx.cn/posts/485): section 二.1
              (standard attention S = QKᵀ, P = softmax(S), O = PV), section 三.2
              (online-softmax update rule), section 三.3 (recomputation).
  [essay]     "当算力不再是瓶颈：重新审视 FlashAttention 的 IO 墙与算法极限"
              (nanhubrain.csdn.net): section 二 (P = softmax(QKᵀ/√d), saved O, m, ℓ),
              section 三.1 (causal mask P_ij = 0 for j > i and the valid-tile set
              S = {(i, j) | j·B_c ≤ i·B_r + B_r − 1}).
  [explainer] "FlashAttention：破解Transformer内存瓶颈的IO感知优化技术"
              (cloud.baidu.com/article/7906313): section "工作原理" (safe softmax
              with the row maximum subtracted), "梯度计算优化" (softmax gradient).

Readings where the pages are silent or garbled are listed per function.
``oracle.dropout`` adds attention with dropout on P (keep decisions from a
Philox4x32-10 counter-based generator, regenerated in the backward).
"""
from .attention import (  # noqa: F401
    allowed_mask,
    forward,
    forward_rows,
    backward,
    backward_rows,
    online_forward,
    merge_partials,
    split_kv_forward,
    causal_tile_set,
    forward_tile_lists,
    backward_tile_lists,
    sampled_forward_backward,
)
from . import dropout  # noqa: F401
