"""B200-native forward pass of MiniMax-Sparse-Attention-style block-sparse
GQA attention: index block scores, per-group Top-k with the current block
kept, and exact sparse softmax attention with LSE.

The computation lives in ``libmsa.so`` (hand-written CUDA for sm_100a, C ABI
in ``include/msa.h``); this package is its Python binding.
"""
from .binding import (EXPORTS, MSA_BF16, MSA_F32, MSA_OK, MSA_WS_FORWARD, MSA_WS_FORWARD_HOST,
                      MSA_WS_SPARSE_ATTN, MsaError, Params, alloc_workspace, forward,
                      forward_with_mass, index_block_scores, make_params, msa_forward,
                      msa_forward_host, msa_forward_mass, msa_query_pieces,
                      msa_sparse_attn_fwd_mass,
                      msa_get_device_error, msa_index_block_scores,
                      msa_kernel_launches, msa_selftest_wait_timeout,
                      msa_sparse_attn_fwd, msa_topk_blocks, msa_workspace_size, params_from,
                      sparse_attn_fwd, status_string, topk_blocks)

__all__ = [
    "EXPORTS", "MSA_BF16", "MSA_F32", "MSA_OK", "MSA_WS_FORWARD", "MSA_WS_FORWARD_HOST",
    "MSA_WS_SPARSE_ATTN", "MsaError", "Params", "alloc_workspace", "forward",
    "forward_with_mass", "index_block_scores", "make_params", "msa_forward", "msa_forward_host",
    "msa_forward_mass", "msa_query_pieces", "msa_sparse_attn_fwd_mass",
    "msa_get_device_error", "msa_index_block_scores", "msa_kernel_launches",
    "msa_selftest_wait_timeout", "msa_sparse_attn_fwd",
    "msa_topk_blocks", "msa_workspace_size", "params_from", "sparse_attn_fwd", "status_string",
    "topk_blocks",
]
