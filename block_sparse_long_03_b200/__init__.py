"""B200-native forward pass of MiniMax-Sparse-Attention-style block-sparse
GQA attention: index block scores, per-group Top-k with the current block
kept, and exact sparse softmax attention with LSE.

The computation lives in ``libmsa.so`` (hand-written CUDA for sm_100a, C ABI
in ``include/msa.h``); this package is its Python binding.  Importing the
package fails when the library has not been built (there is no other
implementation); the library itself is loaded on first use of a binding
name, so that ``block_sparse_long_03_b200.synthetic`` (input generation
only) can be imported without it.
"""
import os as _os

_LIB = _os.path.join(_os.path.dirname(_os.path.abspath(__file__)), "libmsa.so")
if not _os.path.exists(_LIB):
    raise ImportError(f"CUDA library not built: {_LIB} is missing "
                      "(run python block_sparse_long_03_b200/build.py)")

__all__ = [
    "EXPORTS", "MSA_BF16", "MSA_F32", "MSA_OK", "MSA_WS_DECODE_PAGED", "MSA_WS_FORWARD",
    "MSA_WS_INDEX_HIER", "index_hierarchical", "msa_index_hierarchical",
    "MSA_WS_FORWARD_HOST", "MSA_WS_SPARSE_ATTN", "MsaError", "Params", "alloc_workspace",
    "decode_paged", "forward", "msa_decode_paged",
    "forward_with_mass", "index_block_scores", "make_params", "msa_forward", "msa_forward_host",
    "msa_forward_mass", "msa_query_pieces", "msa_sparse_attn_fwd_mass",
    "msa_get_device_error", "msa_index_block_scores", "msa_kernel_launches",
    "msa_selftest_wait_timeout", "msa_sparse_attn_fwd", "msa_profile_begin", "msa_profile_end",
    "msa_bounds_failures",
    "msa_topk_blocks", "msa_workspace_size", "params_from", "sparse_attn_fwd", "status_string",
    "topk_blocks",
]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def __dir__():
    return sorted(list(globals()) + __all__)
