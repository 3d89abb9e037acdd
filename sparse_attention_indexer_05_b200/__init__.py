"""B200 lightning indexer + per-query top-k (dense, dense with the
cutoff-margin adaptive budget, PIVOT Reuse/Refine/block pre-filter, decode,
paged decode, decode with the block pre-filter) and the token-sparse
attention that
consumes the selected positions.

The computation lives in libidx.so (CUDA, sm_100a) behind the C ABI of
include/idx.h; `indexer` is its thin Python binding.
"""
from .indexer import (adaptive_topk, adaptive_workspace_size, debug_decode_scores, debug_scores, decode_block_means,
                      decode_block_minmax, decode_block_topk, decode_block_workspace_size, decode_paged_topk, decode_topk,
                      decode_workspace_size, dense_topk, dense_workspace_size, device_status, pivot_topk,
                      pivot_workspace_size, sparse_attn, uses_tensor_cores)

__all__ = ["dense_topk", "adaptive_topk", "adaptive_workspace_size", "pivot_topk", "decode_topk", "decode_paged_topk",
           "decode_block_means", "decode_block_minmax", "decode_block_topk", "decode_block_workspace_size", "sparse_attn", "dense_workspace_size",
           "pivot_workspace_size", "decode_workspace_size", "device_status", "uses_tensor_cores", "debug_scores",
           "debug_decode_scores"]
