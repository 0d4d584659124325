"""Helpers that compare the CUDA library's outputs with the fp64 oracle.

Tolerances (written here, used by every parity test):
  * block scores and block ids: bit-exact (the index inputs sit on a 1/4 grid
    so every index dot product is exact in fp32 and in fp64);
  * O: max-abs 2e-2 and mean-abs 2e-3 for bf16 I/O, max-abs 1e-4 for fp32;
  * LSE: max-abs 2e-3 for bf16, 1e-5 for fp32 (a stated reading: the
    workload fixes only the O tolerance).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc

TOL = {
    torch.bfloat16: dict(o_max=2e-2, o_mean=2e-3, lse_max=2e-3),
    torch.float32: dict(o_max=1e-4, o_mean=1e-4, lse_max=1e-5),
}


# The KL target's tolerance follows from the LSE tolerance: a slot's mass is a
# head average of exp(lse_slot - lse), and both LSEs are within lse_max of the
# exact value, so |d mass| <= mass * (exp(2 lse_max) - 1) <= 2.01 lse_max.
MASS_TOL = {dt: 2.01 * t["lse_max"] for dt, t in TOL.items()}


def oracle_mass_rows(inp, w, rows, ids_rows, lse_rows):
    """The oracle's KL target [len(rows), G, topk] for sorted `rows`, from the
    kept ids and the oracle's LSE of those rows (as returned by oracle_rows)."""
    rows = np.asarray(sorted(rows), dtype=np.int64)
    out = np.empty(ids_rows.shape, np.float64)
    for b in np.unique(rows // w.T):
        sel = np.nonzero(rows // w.T == b)[0]
        ts = rows[sel] % w.T
        tt = torch.from_numpy(ts)
        Q = inp.Q[int(b)].index_select(0, tt.to(inp.Q.device)).cpu()
        K = inp.K[int(b):int(b) + 1].cpu()
        out[sel] = orc.block_mass(Q, K, ids_rows[sel], lse_rows[sel], ts, T=w.T, block=w.block)
    return out


def oracle_rows(inp, w, rows, *, want_scores=False, ids=None, scale=0.0):
    """Run the oracle for `rows` (r = b * T + t) of the inputs `inp` (device or
    host tensors), with softmax scale `scale` (<= 0: 1/sqrt(d)).  Returns dict
    of numpy arrays indexed like `rows`."""
    rows = np.asarray(sorted(rows), dtype=np.int64)
    T = w.T
    out = {"rows": rows, "ids": [], "O": [], "lse": [], "bs": []}
    by_b = {}
    for r in rows:
        by_b.setdefault(int(r // T), []).append(int(r % T))
    for b, ts in sorted(by_b.items()):
        ts = np.asarray(ts, dtype=np.int64)
        tt = torch.from_numpy(ts)
        k_idx = inp.k_idx[b:b + 1].cpu()
        K = inp.K[b:b + 1].cpu()
        V = inp.V[b:b + 1].cpu()
        q_idx = inp.q_idx[b].index_select(0, tt.to(inp.q_idx.device)).cpu()
        Q = inp.Q[b].index_select(0, tt.to(inp.Q.device)).cpu()
        if ids is None:
            res = orc.forward(q_idx, k_idx, Q, K, V, ts, T=T, block=w.block, topk=w.topk,
                              want_scores=want_scores, scale=scale)
            out["ids"].append(res[0])
            out["O"].append(res[1])
            out["lse"].append(res[2])
            if want_scores:
                out["bs"].append(res[3])
        else:
            id_rows = ids[b].index_select(0, tt.to(ids.device)).cpu().numpy()
            O, lse = orc.attention(Q, K, V, id_rows, ts, T=T, block=w.block, scale=scale)
            out["ids"].append(id_rows)
            out["O"].append(O)
            out["lse"].append(lse)
    for k in ("ids", "O", "lse", "bs"):
        out[k] = np.concatenate(out[k]) if out[k] else None
    return out


def gather_rows(x, rows, T):
    """x [B, T, ...] (device) -> numpy [len(rows), ...] for rows r = b * T + t."""
    flat = x.reshape(x.shape[0] * x.shape[1], *x.shape[2:])
    idx = torch.as_tensor(np.asarray(sorted(rows)), device=x.device)
    return flat.index_select(0, idx).float().cpu().numpy() if x.dtype != torch.int32 else \
        flat.index_select(0, idx).cpu().numpy()


def assert_bits_equal(got, want, where=""):
    """Block scores compared by bit pattern (as float64): -0.0 differs from
    +0.0 here, which a numeric comparison would hide."""
    g = np.ascontiguousarray(got, dtype=np.float64).view(np.int64)
    w = np.ascontiguousarray(want, dtype=np.float64).view(np.int64)
    if not np.array_equal(g, w):
        bad = np.argwhere(g != w)
        r = tuple(bad[0])
        raise AssertionError(f"{where}: block score bits differ at {len(bad)} places; first "
                             f"{r}: got {float(np.asarray(got)[r])!r} want "
                             f"{float(np.asarray(want)[r])!r}")


def assert_ids_equal(got, want, where=""):
    if not np.array_equal(got, want):
        bad = np.argwhere(np.any(got != want, axis=-1))
        r = tuple(bad[0])
        raise AssertionError(f"{where}: block ids differ at {len(bad)} (row, group) pairs; "
                             f"first {r}: got {got[r]} want {want[r]}")


def assert_close(O_gpu, lse_gpu, O_ref, lse_ref, dtype, where=""):
    tol = TOL[dtype]
    dO = np.abs(O_gpu.astype(np.float64) - O_ref)
    dL = np.abs(lse_gpu.astype(np.float64) - lse_ref)
    finite = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), finite), f"{where}: -inf LSE pattern differs"
    dL = dL[finite]
    msg = (f"{where}: O max {dO.max():.3g} (tol {tol['o_max']}), mean {dO.mean():.3g} "
           f"(tol {tol['o_mean']}); LSE max {dL.max() if dL.size else 0:.3g} "
           f"(tol {tol['lse_max']})")
    assert dO.max() <= tol["o_max"] and dO.mean() <= tol["o_mean"], msg
    assert (dL.max() if dL.size else 0.0) <= tol["lse_max"], msg
    return msg
