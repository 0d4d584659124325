"""fp64 CPU oracle for MSA-style block-sparse GQA attention (forward pass).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library never calls it and shares no code with it.

The arithmetic lives in ``msa_oracle.c`` (plain C, fp64, OpenMP over rows),
which follows "MiniMax Sparse Attention -- paper by Lai et al. (2026)",
section "Summary" (index branch, per-group Top-k with the current block
kept, exact softmax over the kept blocks, and the group-averaged Main
Branch distribution the indexer's KL objective matches) and section "Key
points" (k blocks of B_k tokens give k * B_k attended tokens; LSE is a
forward output).  This
module only marshals arrays into that C code.

Every function works on a list of rows ``r = b * T + t`` so that large
shapes can be checked on a sample of rows; query-side arrays are passed
gathered for those rows, key-side arrays whole.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB = os.path.join(_HERE, "libmsa_oracle.so")

F32, BF16 = 0, 1

def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-std=c11", "-Wall", "-shared",
                               "-fPIC", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def bind(path: str):
    """Load a compiled oracle library (the default one, or a variant built
    by a test) and declare its C signatures."""
    lib = ctypes.CDLL(path)
    i64, vp, dbl, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_double, ctypes.c_int
    lib.oracle_block_scores.argtypes = [i64] * 6 + [i32, vp, vp, vp, i64, vp]
    lib.oracle_select_blocks.argtypes = [i64] * 5 + [vp, vp, i64, vp]
    lib.oracle_attention.argtypes = [i64] * 8 + [i32, dbl, vp, vp, vp, vp, vp, i64, vp, vp]
    lib.oracle_forward.argtypes = [i64] * 9 + [i32, dbl] + [vp] * 6 + [i64, vp, vp, vp, vp]
    lib.oracle_block_mass.argtypes = [i64] * 8 + [i32, dbl, vp, vp, vp, vp, vp, i64, vp]
    lib.oracle_forward_paged.argtypes = [i64] * 9 + [i32, dbl, vp, vp, i64, i64, i64] + [vp] * 8
    lib.oracle_select_hierarchical.argtypes = [i64] * 8 + [i32, vp, vp, vp, i64, vp]
    for f in (lib.oracle_block_scores, lib.oracle_select_blocks, lib.oracle_attention,
              lib.oracle_forward, lib.oracle_block_mass, lib.oracle_forward_paged,
              lib.oracle_select_hierarchical, lib.oracle_num_threads):
        f.restype = ctypes.c_int
    return lib


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = bind(build())
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _as_raw(x):
    """Return (contiguous numpy array, dtype code) for fp32 or bf16 data.

    Accepts numpy float32 arrays and CPU torch tensors of dtype float32 or
    bfloat16 (bf16 is passed as its raw 16-bit patterns; the C side widens
    them exactly)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return np.ascontiguousarray(x.view(torch.int16).numpy()), BF16
            if x.dtype == torch.float32:
                return np.ascontiguousarray(x.numpy()), F32
            raise TypeError(f"oracle takes float32 or bfloat16, got {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    raise TypeError(f"oracle takes float32 or bfloat16, got {x.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))


def block_scores(q_idx_rows, k_idx, rows, *, T: int, block: int, lib=None) -> np.ndarray:
    """Block scores [nrows, G, NB] (fp64; -inf for blocks with no causal token).

    q_idx_rows: [nrows, G, d_idx]; k_idx: [B, S, d_idx]."""
    q, dt = _as_raw(q_idx_rows)
    k, dt2 = _as_raw(k_idx)
    assert dt == dt2, "q_idx and k_idx must share a dtype"
    r = _rows(rows)
    nrows, G, d_idx = q.shape
    B, S, _ = k.shape
    NB = -(-S // block)
    out = np.empty((nrows, G, NB), np.float64)
    rc = (lib or _load()).oracle_block_scores(B, T, S, G, d_idx, block, dt, _ptr(q), _ptr(k),
                                     _ptr(r), nrows, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_block_scores failed ({rc})")
    return out


def select_blocks(bs: np.ndarray, rows, *, T: int, S: int, block: int, topk: int,
                  lib=None) -> np.ndarray:
    """Kept block ids [nrows, G, topk] int32, ascending, -1 padded."""
    bs = np.ascontiguousarray(bs, dtype=np.float64)
    r = _rows(rows)
    nrows, G, _ = bs.shape
    ids = np.empty((nrows, G, topk), np.int32)
    rc = (lib or _load()).oracle_select_blocks(T, S, G, block, topk, _ptr(bs), _ptr(r), nrows, _ptr(ids))
    if rc != 0:
        raise ValueError(f"oracle_select_blocks failed ({rc})")
    return ids


def attention(Q_rows, K, V, ids, rows, *, T: int, block: int, scale: float = 0.0, lib=None):
    """(O [nrows, Hq, d], lse [nrows, Hq]) in fp64 over the kept blocks `ids`."""
    q, dt = _as_raw(Q_rows)
    k, dtk = _as_raw(K)
    v, dtv = _as_raw(V)
    assert dt == dtk == dtv, "Q, K and V must share a dtype"
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    r = _rows(rows)
    nrows, Hq, d = q.shape
    B, S, Hkv, _ = k.shape
    topk = ids.shape[-1]
    O = np.empty((nrows, Hq, d), np.float64)
    lse = np.empty((nrows, Hq), np.float64)
    rc = (lib or _load()).oracle_attention(B, T, S, Hq, Hkv, d, block, topk, dt, float(scale),
                                  _ptr(q), _ptr(k), _ptr(v), _ptr(ids), _ptr(r), nrows,
                                  _ptr(O), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_attention failed ({rc})")
    return O, lse


def block_mass(Q_rows, K, ids, lse, rows, *, T: int, block: int, scale: float = 0.0,
               lib=None) -> np.ndarray:
    """Target of the indexer's KL objective: [nrows, G, topk] fp64, the mass
    of each kept slot's block under the row's softmax (normalised by the
    stored `lse` [nrows, Hq]), averaged over the heads of the group."""
    q, dt = _as_raw(Q_rows)
    k, dtk = _as_raw(K)
    assert dt == dtk, "Q and K must share a dtype"
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    r = _rows(rows)
    nrows, Hq, d = q.shape
    B, S, Hkv, _ = k.shape
    topk = ids.shape[-1]
    out = np.empty((nrows, Hkv, topk), np.float64)
    rc = (lib or _load()).oracle_block_mass(B, T, S, Hq, Hkv, d, block, topk, dt, float(scale),
                                            _ptr(q), _ptr(k), _ptr(ids), _ptr(lse), _ptr(r),
                                            nrows, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_block_mass failed ({rc})")
    return out


def forward(q_idx_rows, k_idx, Q_rows, K, V, rows, *, T: int, block: int, topk: int,
            scale: float = 0.0, want_scores: bool = False, lib=None):
    """Whole forward pass for the given rows: (ids, O, lse[, bs])."""
    qi, dt = _as_raw(q_idx_rows)
    ki, _ = _as_raw(k_idx)
    q, _ = _as_raw(Q_rows)
    k, _ = _as_raw(K)
    v, _ = _as_raw(V)
    r = _rows(rows)
    nrows, Hq, d = q.shape
    B, S, Hkv, _ = k.shape
    d_idx = qi.shape[-1]
    NB = -(-S // block)
    ids = np.empty((nrows, Hkv, topk), np.int32)
    O = np.empty((nrows, Hq, d), np.float64)
    lse = np.empty((nrows, Hq), np.float64)
    bs = np.empty((nrows, Hkv, NB), np.float64) if want_scores else None
    rc = (lib or _load()).oracle_forward(B, T, S, Hq, Hkv, d, d_idx, block, topk, dt, float(scale),
                                _ptr(qi), _ptr(ki), _ptr(q), _ptr(k), _ptr(v), _ptr(r), nrows,
                                _ptr(ids), _ptr(O), _ptr(lse),
                                _ptr(bs) if bs is not None else None)
    if rc != 0:
        raise ValueError(f"oracle_forward failed ({rc})")
    return (ids, O, lse, bs) if want_scores else (ids, O, lse)


def forward_paged(q_idx, k_idx_cache, Q, K_cache, V_cache, seq_lens, block_table, *, S: int,
                  block: int, topk: int, scale: float = 0.0, lib=None):
    """Forward pass over a paged cache with per-sequence lengths:
    (ids [B, T, G, topk], O [B, T, Hq, d], lse [B, T, Hq]).

    q_idx [B, T, G, d_idx]; k_idx_cache [num_pages, page_size, d_idx];
    Q [B, T, Hq, d]; K_cache, V_cache [num_pages, page_size, Hkv, d];
    seq_lens [B] and block_table [B, max_pages] int32 (host); S the capacity."""
    qi, dt = _as_raw(q_idx)
    ki, _ = _as_raw(k_idx_cache)
    q, _ = _as_raw(Q)
    k, _ = _as_raw(K_cache)
    v, _ = _as_raw(V_cache)
    lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32).reshape(-1))
    table = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    B, T, Hq, d = q.shape
    num_pages, page_size, Hkv, _ = k.shape
    d_idx = qi.shape[-1]
    max_pages = table.shape[1]
    ids = np.empty((B, T, Hkv, topk), np.int32)
    O = np.empty((B, T, Hq, d), np.float64)
    lse = np.empty((B, T, Hq), np.float64)
    rc = (lib or _load()).oracle_forward_paged(
        B, T, S, Hq, Hkv, d, d_idx, block, topk, dt, float(scale), _ptr(lens), _ptr(table),
        page_size, max_pages, num_pages, _ptr(qi), _ptr(ki), _ptr(q), _ptr(k), _ptr(v),
        _ptr(ids), _ptr(O), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_forward_paged failed ({rc})")
    return ids, O, lse


def select_hierarchical(q_idx_rows, k_idx, rows, *, T: int, block: int, topk: int, kc: int,
                        lib=None) -> np.ndarray:
    """Coarse-to-fine block selection: ids [nrows, G, topk] int32 (ascending,
    -1 padded).  Coarse: index query . the block's mean index key; the kc - 1
    best earlier blocks are the candidates; fine: their exact max-pooled
    scores; kept: the current block and the topk - 1 best candidates."""
    q, dt = _as_raw(q_idx_rows)
    k, dt2 = _as_raw(k_idx)
    assert dt == dt2, "q_idx and k_idx must share a dtype"
    r = _rows(rows)
    nrows, G, d_idx = q.shape
    B, S, _ = k.shape
    ids = np.empty((nrows, G, topk), np.int32)
    rc = (lib or _load()).oracle_select_hierarchical(B, T, S, G, d_idx, block, topk, kc, dt,
                                                     _ptr(q), _ptr(k), _ptr(r), nrows, _ptr(ids))
    if rc != 0:
        raise ValueError(f"oracle_select_hierarchical failed ({rc})")
    return ids
