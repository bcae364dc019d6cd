"""CPU oracle for the BA-Att hot path.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, obviously-correct
NumPy restatement of what the GPU library computes. It exists to check the
CUDA path, never to stand in for it: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py`` may import it. The
product path (``block_sparse_attention_ba_b200``) never imports it, and the two
share no code; they meet only in the seeded input generators, which hold none
of the method's arithmetic.

Sources (cited by page title and section throughout):

* [BA-Att]  "Efficient Long-Context Modeling in Diffusion Language Models via
  Block Approximate Sparse Attention" (arXiv 2605.19726): abstract, "The pith",
  "Core claim", "What carries the argument", Figure 2 caption, referee report.
* [FlashBlock]  "FlashBlock: Attention Caching for Efficient Long-Context Block
  Diffusion" (arXiv 2602.05305): the attention decomposition (Eq. 5) and the
  log-space composition of cached and fresh partial attentions (Eq. 9).

The pages state the ingredients of the selector in prose only (block-wise
pre-downsampling, per-dimension diagonal Q/K variances, a covariance-compensated
correction, norm sorting keeping a top fraction). Every formula below is the
plain reading of that prose, stated in the docstring of the function that
implements it.

Parity status: every public function is pinned by tests in
``tests/test_oracle.py``. The two diagnostics (``spearman_vs_post`` and
``topk_recall_vs_post``) have no value on the pages; they are pinned to a
library routine, closed forms and brute force instead.
"""

from .ba_att_oracle import (  # noqa: F401
    num_blocks,
    block_counts,
    keep_count,
    block_stats,
    corrected_scores,
    pooled_scores,
    pre_downsample_map,
    select_topk,
    selection_scores,
    select_by_mass,
    mass_share_before,
    near_tie_mask,
    masked_attention,
    block_rows_attention,
    dense_attention,
    merge_lse,
    split_lists,
    complement_lists,
    post_downsample_map,
    block_mass_via_lse,
    spearman_vs_post,
    topk_recall_vs_post,
)
