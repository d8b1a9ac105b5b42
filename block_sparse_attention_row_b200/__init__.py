"""Hybrid Top-k+Top-p block-sparse attention for NVIDIA B200 (sm_100a).

The compute lives in libsparse_attn.so (C ABI: include/sparse_attn.h); this
package is its Python binding. Build the library with ``build.build()``.
"""
from .capi import (EXPORTED, SparseAttnError, bwd_workspace_bytes, check_device_error, host_workspace_bytes,
                   load_library, mask_workspace_bytes, num_blocks, sparse_attn, sparse_attn_fwd,
                   sparse_attn_bwd, sparse_attn_fwd_dense, sparse_attn_host, sparse_attn_mask,
                   sparse_attn_select, sparse_attn_quantize_fp8, sparse_attn_fwd_fp8,
                   sparse_attn_sparse_linear, sparse_linear_workspace_bytes, kmeans_workspace_bytes,
                   sparse_attn_kmeans_permutation, sparse_attn_permute_rows,
                   permuted_sparse_attn, fused_workspace_bytes, sparse_attn_fused, version)

from .sharding import head_range, head_shard

__all__ = ["head_range", "head_shard", "EXPORTED", "SparseAttnError", "bwd_workspace_bytes", "check_device_error", "sparse_attn_bwd", "host_workspace_bytes",
           "load_library", "mask_workspace_bytes", "num_blocks", "sparse_attn", "sparse_attn_fwd",
           "sparse_attn_fwd_dense", "sparse_attn_host", "sparse_attn_mask", "sparse_attn_select",
           "sparse_attn_quantize_fp8", "sparse_attn_fwd_fp8", "sparse_attn_sparse_linear",
           "sparse_linear_workspace_bytes", "kmeans_workspace_bytes", "sparse_attn_kmeans_permutation",
           "sparse_attn_permute_rows", "permuted_sparse_attn", "fused_workspace_bytes", "sparse_attn_fused",
           "version"]
