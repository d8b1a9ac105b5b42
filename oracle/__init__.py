"""CPU oracle for hybrid Top-k+Top-p block-sparse attention.

TEST INFRASTRUCTURE ONLY. This package is the plain, slow, fp64 statement of
what the sparse-attention path computes, used to check the CUDA path. Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline``
leg and its ``--impl reference`` arm) may import or call it. The product
package ``block_sparse_attention_row_b200`` never imports it and has no CPU
fallback; the oracle shares no code with it.

Sources (gist.science summaries; cited by page title and section):

* "SpargeAttention2: Trainable Sparse Attention via Hybrid Top-k+Top-p
  Masking and Distillation Fine-Tuning" (Hindi and Arabic summaries):
  §1 Problem Statement (the Top-k and Top-p rules and their failure modes),
  §2A Hybrid Top-k + Top-p Masking (per-row union), §2C Efficient Kernel
  Implementation (block-level mask over tiles, masked tiles skipped), and
  §2B Velocity Distillation Fine-Tuning (the sparse attention is trained
  through, hence its backward pass in ``sparse_attn_backward``).
* "SLA2: Sparse-Linear Attention with Learnable Routing and QAT": §1 Problem
  Statement and §2B Learnable Router (a compressed score computed from pooled
  queries and keys), §2A Faithful Sparse-Linear Formulation (the alpha mix of
  a sparse and a linear branch: ``sparse_linear_oracle``) and §2C
  Quantization-Aware Training (the low-bit sparse branch: ``sparse_attn_fp8``).
* "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via
  Semantic-Aware Permutation": §1 (mean or max pooling of contiguous token
  blocks), §2A Semantic-Aware Permutation (k-means clustering and reordering of
  the tokens: ``svg_permutation_oracle``) and §2B Centroid-Based Top-p Selection (sort by score, take items
  until the cumulative score reaches p).

Parity pins: every forward function here is pinned by
``tests/test_oracle_pins.py`` (closed forms, hand rows under ``tests/golden/``,
invariants, library special cases, brute force on tiny inputs), the backward
pass by ``tests/test_oracle_backward.py``. The absolute values of the score matrix
and of the output on the synthetic workloads have no printed counterpart on
the pages; beyond those pins they are fixed only by the definitions.
"""
from .sparse_attn_oracle import (
    to_f64,
    pool_blocks,
    block_scores,
    topk_count,
    topp_threshold,
    select_row,
    hybrid_select,
    hybrid_mask,
    attend_row,
    block_sparse_attention,
    row_sample,
)
from .sparse_attn_backward import attend_row_backward, block_sparse_attention_backward
from .sparse_attn_fp8 import (block_sparse_attention_fp8, dequantize_blocks, e4m3_round,
                              quantize_blocks)
from .sparse_linear_oracle import linear_row, phi, sparse_linear_attention
from .svg_permutation_oracle import kmeans_permutation, permuted_sparse_attention

__all__ = [
    "to_f64", "pool_blocks", "block_scores", "topk_count", "topp_threshold",
    "select_row", "hybrid_select", "hybrid_mask", "attend_row",
    "block_sparse_attention", "row_sample", "attend_row_backward",
    "block_sparse_attention_backward", "e4m3_round", "quantize_blocks", "dequantize_blocks",
    "block_sparse_attention_fp8", "phi", "linear_row", "sparse_linear_attention",
    "kmeans_permutation", "permuted_sparse_attention",
]
