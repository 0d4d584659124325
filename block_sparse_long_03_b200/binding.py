"""Thin Python binding of the C ABI in ``include/msa.h``.

Argument marshalling only: every function takes torch CUDA tensors, checks
dtypes and shapes, and passes raw device pointers plus the current CUDA
stream to ``libmsa.so``.  All computation happens in the library's CUDA
kernels.  If the library is missing the import fails loudly; there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MSA_LIBRARY=checked selects the bounds-checked build (libmsa_checked.so)
LIB_PATH = os.path.join(_HERE, "libmsa_checked.so" if os.environ.get("MSA_LIBRARY") == "checked"
                        else "libmsa.so")

MSA_OK = 0
MSA_F32, MSA_BF16 = 0, 1
MSA_WS_SPARSE_ATTN, MSA_WS_FORWARD, MSA_WS_FORWARD_HOST, MSA_WS_DECODE_PAGED = 0, 1, 2, 3
MSA_WS_INDEX_HIER = 4
STATUS_NAMES = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_CUDA",
                4: "MSA_ERR_DEVICE_TIMEOUT", 5: "MSA_ERR_WORKSPACE", 6: "MSA_ERR_BAD_BLOCK_IDS",
                7: "MSA_ERR_BAD_PAGE_TABLE"}

# Every symbol the header declares (checked by the CPU test suite).
EXPORTS = ("msa_status_string", "msa_index_block_scores", "msa_topk_blocks",
           "msa_workspace_size", "msa_sparse_attn_fwd", "msa_forward", "msa_get_device_error",
           "msa_kernel_launches", "msa_forward_noalloc", "msa_forward_host",
           "msa_selftest_wait_timeout", "msa_sparse_attn_fwd_mass", "msa_forward_mass",
           "msa_query_pieces", "msa_decode_paged", "msa_index_hierarchical",
           "msa_bounds_failures", "msa_profile_begin", "msa_profile_end")


class MsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class Params(ctypes.Structure):
    """msa_params_t."""
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "T", "S", "Hq", "Hkv", "d", "d_idx", "block", "topk", "dtype")] + \
               [("scale", ctypes.c_float)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library not built: {LIB_PATH} is missing "
                          "(run python block_sparse_long_03_b200/build.py)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, P = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(Params)
    st = ctypes.c_int
    lib.msa_status_string.argtypes = [st]
    lib.msa_status_string.restype = ctypes.c_char_p
    lib.msa_index_block_scores.argtypes = [P, vp, vp, vp, vp]
    lib.msa_topk_blocks.argtypes = [P, vp, vp, vp]
    lib.msa_workspace_size.argtypes = [P, ctypes.c_int]
    lib.msa_workspace_size.restype = sz
    lib.msa_sparse_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_get_device_error.argtypes = [vp, vp]
    lib.msa_forward_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.msa_forward_noalloc.restype = st
    lib.msa_forward_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_forward_host.restype = st
    lib.msa_sparse_attn_fwd_mass.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_sparse_attn_fwd_mass.restype = st
    lib.msa_forward_mass.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_forward_mass.restype = st
    i32 = ctypes.c_int32
    lib.msa_decode_paged.argtypes = [P, vp, vp, i32, i32, i32] + [vp] * 8 + [vp, sz, vp]
    lib.msa_decode_paged.restype = st
    lib.msa_index_hierarchical.argtypes = [P, i32, vp, vp, vp, vp, sz, vp]
    lib.msa_index_hierarchical.restype = st
    lib.msa_query_pieces.argtypes = [P, ctypes.c_int, vp, ctypes.c_int64]
    lib.msa_query_pieces.restype = ctypes.c_int64
    lib.msa_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint32, vp]
    lib.msa_selftest_wait_timeout.restype = st
    lib.msa_kernel_launches.argtypes = []
    lib.msa_kernel_launches.restype = ctypes.c_uint64
    lib.msa_bounds_failures.argtypes = []
    lib.msa_bounds_failures.restype = ctypes.c_uint32
    lib.msa_profile_begin.argtypes = []
    lib.msa_profile_begin.restype = st
    lib.msa_profile_end.argtypes = [vp, vp, vp, vp]
    lib.msa_profile_end.restype = st
    for name in ("msa_index_block_scores", "msa_topk_blocks", "msa_sparse_attn_fwd",
                 "msa_forward", "msa_get_device_error"):
        getattr(lib, name).restype = st
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.msa_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != MSA_OK:
        raise MsaError(status, where)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_params(*, B, T, S, Hq, Hkv, d, d_idx, block, topk, dtype, scale=0.0) -> Params:
    code = {torch.float32: MSA_F32, torch.bfloat16: MSA_BF16}[dtype]
    return Params(B, T, S, Hq, Hkv, d, d_idx, block, topk, code, float(scale))


def params_from(q_idx, Q, K, *, block: int, topk: int, scale: float = 0.0) -> Params:
    B, T, Hq, d = Q.shape
    S, Hkv = K.shape[1], K.shape[2]
    return make_params(B=B, T=T, S=S, Hq=Hq, Hkv=Hkv, d=d, d_idx=q_idx.shape[-1], block=block,
                       topk=topk, dtype=Q.dtype, scale=scale)


def msa_workspace_size(params: Params, which: int) -> int:
    return int(lib.msa_workspace_size(ctypes.byref(params), int(which)))


def alloc_workspace(params: Params, which: int, device=None) -> torch.Tensor:
    n = msa_workspace_size(params, which)
    if n == 0:
        raise MsaError(1, "msa_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def msa_index_block_scores(params: Params, q_idx, k_idx, block_scores, stream=None):
    _check(lib.msa_index_block_scores(ctypes.byref(params), _ptr(q_idx), _ptr(k_idx),
                                      _ptr(block_scores), _stream(stream)),
           "msa_index_block_scores")


def msa_topk_blocks(params: Params, block_scores, block_ids, stream=None):
    _check(lib.msa_topk_blocks(ctypes.byref(params), _ptr(block_scores), _ptr(block_ids),
                               _stream(stream)), "msa_topk_blocks")


def msa_sparse_attn_fwd(params: Params, Q, K, V, block_ids, O, lse, workspace, stream=None):
    _check(lib.msa_sparse_attn_fwd(ctypes.byref(params), _ptr(Q), _ptr(K), _ptr(V),
                                   _ptr(block_ids), _ptr(O), _ptr(lse), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "msa_sparse_attn_fwd")


def msa_forward(params: Params, q_idx, k_idx, Q, K, V, block_ids, O, lse, workspace,
                stream=None):
    _check(lib.msa_forward(ctypes.byref(params), _ptr(q_idx), _ptr(k_idx), _ptr(Q), _ptr(K),
                           _ptr(V), _ptr(block_ids), _ptr(O), _ptr(lse), _ptr(workspace),
                           workspace.numel(), _stream(stream)), "msa_forward")


def msa_sparse_attn_fwd_mass(params: Params, Q, K, V, block_ids, O, lse, block_mass, workspace,
                             stream=None):
    """msa_sparse_attn_fwd plus block_mass [B, T, G, topk] fp32: each kept slot's share of
    the row's softmax averaged over the group's heads (the indexer's KL target)."""
    _check(lib.msa_sparse_attn_fwd_mass(ctypes.byref(params), _ptr(Q), _ptr(K), _ptr(V),
                                        _ptr(block_ids), _ptr(O), _ptr(lse), _ptr(block_mass),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
           "msa_sparse_attn_fwd_mass")


def msa_forward_mass(params: Params, q_idx, k_idx, Q, K, V, block_ids, O, lse, block_mass,
                     workspace, stream=None):
    """msa_forward plus block_mass (see msa_sparse_attn_fwd_mass)."""
    _check(lib.msa_forward_mass(ctypes.byref(params), _ptr(q_idx), _ptr(k_idx), _ptr(Q),
                                _ptr(K), _ptr(V), _ptr(block_ids), _ptr(O), _ptr(lse),
                                _ptr(block_mass), _ptr(workspace), workspace.numel(),
                                _stream(stream)), "msa_forward_mass")


def msa_forward_host(params: Params, q_idx, k_idx, Q, K, V, block_ids, O, lse, device_buffer,
                     stream=None):
    """msa_forward on page-locked host tensors (``pin_memory()``); the copies to
    and from ``device_buffer`` (a CUDA uint8 tensor of at least
    ``msa_workspace_size(params, MSA_WS_FORWARD_HOST)`` bytes) run inside the
    call, overlapped with the kernels.  O, lse and block_ids are valid once
    ``stream`` has passed the call."""
    _check(lib.msa_forward_host(ctypes.byref(params), _ptr(q_idx), _ptr(k_idx), _ptr(Q),
                                _ptr(K), _ptr(V), _ptr(block_ids), _ptr(O), _ptr(lse),
                                _ptr(device_buffer), device_buffer.numel(), _stream(stream)),
           "msa_forward_host")


def msa_decode_paged(params: Params, seq_lens, block_table, page_size: int, num_pages: int,
                     q_idx, k_idx_cache, Q, K_cache, V_cache, block_ids, O, lse, workspace,
                     stream=None):
    """Decode steps over a paged cache: seq_lens [B] and block_table
    [B, max_pages] int32 CUDA tensors; caches [num_pages, page_size, ...]."""
    _check(lib.msa_decode_paged(ctypes.byref(params), _ptr(seq_lens), _ptr(block_table),
                                int(page_size), int(block_table.shape[1]), int(num_pages),
                                _ptr(q_idx), _ptr(k_idx_cache), _ptr(Q), _ptr(K_cache),
                                _ptr(V_cache), _ptr(block_ids), _ptr(O), _ptr(lse),
                                _ptr(workspace), workspace.numel(), _stream(stream)),
           "msa_decode_paged")


def msa_index_hierarchical(params: Params, kc: int, q_idx, k_idx, block_ids, workspace,
                           stream=None):
    """Coarse-to-fine block selection (block means, kc candidates, exact
    rescoring) into block_ids [B, T, G, topk]."""
    _check(lib.msa_index_hierarchical(ctypes.byref(params), int(kc), _ptr(q_idx), _ptr(k_idx),
                                      _ptr(block_ids), _ptr(workspace), workspace.numel(),
                                      _stream(stream)), "msa_index_hierarchical")


def msa_get_device_error(workspace, stream=None) -> int:
    """The status recorded on the device by the last call that used `workspace`."""
    return int(lib.msa_get_device_error(_ptr(workspace), _stream(stream)))


def msa_selftest_wait_timeout(workspace, limit_us: int, stream=None):
    """Run the device wait-timeout check (see include/msa.h)."""
    _check(lib.msa_selftest_wait_timeout(_ptr(workspace), workspace.numel(), int(limit_us),
                                         _stream(stream)), "msa_selftest_wait_timeout")


def msa_query_pieces(params: Params, which: int) -> list:
    """The (sequence, first query, end query) pieces a call splits its work into
    (which = MSA_WS_FORWARD or MSA_WS_FORWARD_HOST); sequence -1 means all."""
    n = int(lib.msa_query_pieces(ctypes.byref(params), int(which), None, 0))
    if n <= 0:
        return []
    buf = (ctypes.c_int32 * (3 * n))()
    lib.msa_query_pieces(ctypes.byref(params), int(which), buf, n)
    return [tuple(buf[3 * i:3 * i + 3]) for i in range(n)]


def msa_kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib.msa_kernel_launches())


def msa_bounds_failures() -> int:
    """Failed device bounds checks since load (checked build; 0 otherwise)."""
    return int(lib.msa_bounds_failures())


def msa_profile_begin():
    _check(lib.msa_profile_begin(), "msa_profile_begin")


def msa_profile_end() -> dict:
    """Summed device time (ms) and launch counts of the tensor-core attention
    and merge kernels launched since msa_profile_begin."""
    am, mm = ctypes.c_double(0.0), ctypes.c_double(0.0)
    an, mn = ctypes.c_int64(0), ctypes.c_int64(0)
    _check(lib.msa_profile_end(ctypes.byref(am), ctypes.byref(an), ctypes.byref(mm),
                               ctypes.byref(mn)), "msa_profile_end")
    return {"attn_ms": am.value, "attn_launches": an.value, "merge_ms": mm.value,
            "merge_launches": mn.value}


# ---- convenience wrappers that allocate outputs with torch ----------------

def index_block_scores(q_idx, k_idx, *, block: int, T: int | None = None):
    B, T_, G, d_idx = q_idx.shape
    S = k_idx.shape[1]
    p = make_params(B=B, T=T_, S=S, Hq=G, Hkv=G, d=64, d_idx=d_idx, block=block, topk=1,
                    dtype=q_idx.dtype)
    bs = torch.empty((B, T_, G, S // block), dtype=torch.float32, device=q_idx.device)
    msa_index_block_scores(p, q_idx, k_idx, bs)
    return bs


def topk_blocks(block_scores, *, S: int, block: int, topk: int):
    B, T, G, NB = block_scores.shape
    p = make_params(B=B, T=T, S=S, Hq=G, Hkv=G, d=64, d_idx=16, block=block, topk=topk,
                    dtype=torch.float32)
    ids = torch.empty((B, T, G, topk), dtype=torch.int32, device=block_scores.device)
    msa_topk_blocks(p, block_scores, ids)
    return ids


def sparse_attn_fwd(Q, K, V, block_ids, *, block: int, scale: float = 0.0):
    B, T, Hq, d = Q.shape
    S, Hkv = K.shape[1], K.shape[2]
    p = make_params(B=B, T=T, S=S, Hq=Hq, Hkv=Hkv, d=d, d_idx=16, block=block,
                    topk=block_ids.shape[-1], dtype=Q.dtype, scale=scale)
    O = torch.empty_like(Q)
    lse = torch.empty((B, T, Hq), dtype=torch.float32, device=Q.device)
    ws = alloc_workspace(p, MSA_WS_SPARSE_ATTN, Q.device)
    msa_sparse_attn_fwd(p, Q, K, V, block_ids, O, lse, ws)
    return O, lse, ws


def forward(q_idx, k_idx, Q, K, V, *, block: int, topk: int, scale: float = 0.0):
    """The whole forward pass; returns (O, lse, block_ids, workspace)."""
    p = params_from(q_idx, Q, K, block=block, topk=topk, scale=scale)
    O = torch.empty_like(Q)
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=Q.device)
    ids = torch.empty((*Q.shape[:2], K.shape[2], topk), dtype=torch.int32, device=Q.device)
    ws = alloc_workspace(p, MSA_WS_FORWARD, Q.device)
    msa_forward(p, q_idx, k_idx, Q, K, V, ids, O, lse, ws)
    return O, lse, ids, ws


def forward_with_mass(q_idx, k_idx, Q, K, V, *, block: int, topk: int, scale: float = 0.0):
    """The whole forward pass plus the indexer's KL target; returns
    (O, lse, block_ids, block_mass, workspace)."""
    p = params_from(q_idx, Q, K, block=block, topk=topk, scale=scale)
    O = torch.empty_like(Q)
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=Q.device)
    ids = torch.empty((*Q.shape[:2], K.shape[2], topk), dtype=torch.int32, device=Q.device)
    mass = torch.empty((*Q.shape[:2], K.shape[2], topk), dtype=torch.float32, device=Q.device)
    ws = alloc_workspace(p, MSA_WS_FORWARD, Q.device)
    msa_forward_mass(p, q_idx, k_idx, Q, K, V, ids, O, lse, mass, ws)
    return O, lse, ids, mass, ws


def decode_paged(q_idx, k_idx_cache, Q, K_cache, V_cache, seq_lens, block_table, *, S: int,
                 block: int, topk: int, scale: float = 0.0):
    """Decode steps over a paged KV cache with per-sequence lengths; returns
    (O, lse, block_ids, workspace).  S is the capacity (a multiple of block,
    at most block_table.shape[1] * page_size)."""
    B, T, Hq, d = Q.shape
    num_pages, page_size, Hkv, _ = K_cache.shape
    p = make_params(B=B, T=T, S=S, Hq=Hq, Hkv=Hkv, d=d, d_idx=q_idx.shape[-1], block=block,
                    topk=topk, dtype=Q.dtype, scale=scale)
    O = torch.empty_like(Q)
    lse = torch.empty((B, T, Hq), dtype=torch.float32, device=Q.device)
    ids = torch.empty((B, T, Hkv, topk), dtype=torch.int32, device=Q.device)
    ws = alloc_workspace(p, MSA_WS_DECODE_PAGED, Q.device)
    msa_decode_paged(p, seq_lens, block_table, page_size, num_pages, q_idx, k_idx_cache, Q,
                     K_cache, V_cache, ids, O, lse, ws)
    return O, lse, ids, ws


def index_hierarchical(q_idx, k_idx, *, block: int, topk: int, kc: int):
    """Coarse-to-fine block selection; returns (block_ids, workspace)."""
    B, T, G, d_idx = q_idx.shape
    S = k_idx.shape[1]
    p = make_params(B=B, T=T, S=S, Hq=G, Hkv=G, d=64, d_idx=d_idx, block=block, topk=topk,
                    dtype=q_idx.dtype)
    ids = torch.empty((B, T, G, topk), dtype=torch.int32, device=q_idx.device)
    ws = alloc_workspace(p, MSA_WS_INDEX_HIER, q_idx.device)
    msa_index_hierarchical(p, kc, q_idx, k_idx, ids, ws)
    return ids, ws
