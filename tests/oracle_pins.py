"""Pins of the fp64 oracle to things other than itself.

Each ``pin_*`` function takes a compiled oracle library handle (the real one,
or a deliberately broken variant built by the mutation test) and raises
AssertionError when the oracle disagrees with what the method's definition
and mathematics fix:

* brute force: the full token score matrix from a library matmul, max-pooled
  by reshaping, and the kept set decided by COUNTING better candidates (no
  sort), for tiny inputs ("MiniMax Sparse Attention", Summary: max-pooled
  token-level index scores, per-group Top-k, current block kept);
* the dense limit: with every causal block kept, the output is dense causal
  GQA attention, computed by torch's scaled_dot_product_attention in fp64;
* masked attention: for any kept set, the output is scaled_dot_product_attention
  with a boolean mask that allows exactly the kept blocks' causal tokens;
* closed forms and invariants: all-equal index scores keep blocks
  {0..k-2} plus the current one; constant values give a constant output; a
  single attended key gives that key's value; LSE brackets;
* exactness of the inputs' grid: bf16 and fp32 copies of the same grid
  values give bit-identical oracle results;
* the indexer's KL target (Summary: the indexer matches the group-averaged
  Main Branch distribution): torch's masked softmax summed per block and
  averaged over the group's heads, sum-to-one, and the equal-scores share.

Inputs are small (a few hundred tokens) so every pin runs in well under a
second on CPU.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc


def _grid(rng, shape):
    return (rng.integers(-4, 5, size=shape).astype(np.float32) / 4.0)


def brute_block_scores(q_idx, k_idx, T, block):
    """[B, T, G, NB] block scores from a full fp64 score matrix (numpy)."""
    B, _, G, _ = q_idx.shape
    S = k_idx.shape[1]
    NB = -(-S // block)
    s = np.einsum("btgi,bji->btgj", q_idx.astype(np.float64), k_idx.astype(np.float64))
    pos = S - T + np.arange(T)
    causal = np.arange(S)[None, :] <= pos[:, None]            # [T, S]
    s = np.where(causal[None, :, None, :], s, -np.inf)
    pad = NB * block - S
    s = np.concatenate([s, np.full(s.shape[:-1] + (pad,), -np.inf)], axis=-1)
    return s.reshape(B, T, G, NB, block).max(axis=-1)


def brute_kept_sets(bs_row, cb, k):
    """Kept set by counting: n < cb is kept iff fewer than k-1 candidates
    beat it (higher score, or equal score and lower id)."""
    kept = {cb}
    for n in range(cb):
        better = sum(1 for m in range(cb)
                     if bs_row[m] > bs_row[n] or (bs_row[m] == bs_row[n] and m < n))
        if better < k - 1:
            kept.add(n)
    return kept


def _rows_all(B, T):
    return np.arange(B * T, dtype=np.int64)


def pin_brute_force_selection(lib):
    rng = np.random.default_rng(7)
    cases = [  # B, T, S, G, d_idx, block, k
        (2, 96, 96, 2, 4, 16, 3),
        (1, 40, 200, 3, 4, 16, 5),     # T < S (bottom-right alignment), S % block != 0
        (1, 64, 64, 1, 8, 8, 8),
    ]
    for B, T, S, G, d_idx, block, k in cases:
        q = _grid(rng, (B, T, G, d_idx))
        kk = _grid(rng, (B, S, d_idx))
        rows = _rows_all(B, T)
        bs = orc.block_scores(q.reshape(B * T, G, d_idx), kk, rows, T=T, block=block, lib=lib)
        ref = brute_block_scores(q, kk, T, block).reshape(B * T, G, -1)
        assert np.array_equal(bs, ref), "block scores differ from brute force"
        ids = orc.select_blocks(bs, rows, T=T, S=S, block=block, topk=k, lib=lib)
        for ri in range(B * T):
            t = ri % T
            cb = (S - T + t) // block
            for g in range(G):
                want = brute_kept_sets(ref[ri, g], cb, k)
                got = ids[ri, g]
                n_kept = min(k, cb + 1)
                assert list(got[:n_kept]) == sorted(want), (ri, g, got, sorted(want))
                assert np.all(got[n_kept:] == -1)


def _sdpa_reference(Q, K, V, allowed, scale):
    """O and LSE by torch scaled_dot_product_attention (fp64) with a boolean
    mask allowed [B, T, Hq, S]; GQA by repeating each KV head over its group."""
    B, T, Hq, d = Q.shape
    Hkv = K.shape[2]
    R = Hq // Hkv
    q = torch.from_numpy(Q.astype(np.float64)).permute(0, 2, 1, 3)          # B Hq T d
    k = torch.from_numpy(K.astype(np.float64)).permute(0, 2, 1, 3).repeat_interleave(R, dim=1)
    v = torch.from_numpy(V.astype(np.float64)).permute(0, 2, 1, 3).repeat_interleave(R, dim=1)
    m = torch.from_numpy(allowed).permute(0, 2, 1, 3)                      # B Hq T S
    O = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)
    s = (q @ k.transpose(-1, -2)) * scale
    lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    return O.permute(0, 2, 1, 3).numpy(), lse.permute(0, 2, 1).numpy()


def _allowed_from_ids(ids, B, T, S, Hq, Hkv, block):
    """Boolean [B, T, Hq, S]: token j allowed iff its block is kept and j <= p(t)."""
    R = Hq // Hkv
    allowed = np.zeros((B, T, Hq, S), dtype=bool)
    tok_block = np.arange(S) // block
    for b in range(B):
        for t in range(T):
            p = S - T + t
            for h in range(Hq):
                kept = [n for n in ids[b * T + t, h // R] if n >= 0]
                allowed[b, t, h] = np.isin(tok_block, kept) & (np.arange(S) <= p)
    return allowed


def pin_dense_limit(lib):
    rng = np.random.default_rng(11)
    for B, T, S, Hq, Hkv, d, block in [(1, 48, 48, 4, 2, 8, 8), (2, 20, 70, 6, 3, 16, 16)]:
        NB = -(-S // block)
        Q = rng.standard_normal((B, T, Hq, d)).astype(np.float32)
        K = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
        V = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
        rows = _rows_all(B, T)
        ids = np.tile(np.arange(NB, dtype=np.int32), (B * T, Hkv, 1))     # every block kept
        O, lse = orc.attention(Q.reshape(B * T, Hq, d), K, V, ids, rows, T=T, block=block, lib=lib)
        allowed = _allowed_from_ids(ids, B, T, S, Hq, Hkv, block)
        pos = S - T + np.arange(T)
        dense = np.arange(S)[None, :] <= pos[:, None]
        assert np.array_equal(allowed, np.broadcast_to(dense[None, :, None, :], allowed.shape))
        O_ref, lse_ref = _sdpa_reference(Q, K, V, allowed, 1.0 / np.sqrt(d))
        np.testing.assert_allclose(O, O_ref.reshape(B * T, Hq, d), rtol=0, atol=1e-10)
        np.testing.assert_allclose(lse, lse_ref.reshape(B * T, Hq), rtol=0, atol=1e-10)
        # the whole pass with k >= NB is dense causal attention too
        q_idx = _grid(rng, (B * T, Hkv, 4))
        k_idx = _grid(rng, (B, S, 4))
        ids2, O2, lse2 = orc.forward(q_idx, k_idx, Q.reshape(B * T, Hq, d), K, V, rows, T=T,
                                     block=block, topk=NB, lib=lib)
        np.testing.assert_allclose(O2, O_ref.reshape(B * T, Hq, d), rtol=0, atol=1e-10)
        np.testing.assert_allclose(lse2, lse_ref.reshape(B * T, Hq), rtol=0, atol=1e-10)


def pin_masked_attention(lib):
    """Sparse kept sets: equal to SDPA with the kept-block mask."""
    rng = np.random.default_rng(13)
    B, T, S, Hq, Hkv, d, d_idx, block, k = 1, 64, 64, 4, 2, 16, 4, 8, 3
    Q = rng.standard_normal((B, T, Hq, d)).astype(np.float32)
    K = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
    q_idx = _grid(rng, (B * T, Hkv, d_idx))
    k_idx = _grid(rng, (B, S, d_idx))
    rows = _rows_all(B, T)
    ids, O, lse = orc.forward(q_idx, k_idx, Q.reshape(B * T, Hq, d), K, V, rows, T=T,
                              block=block, topk=k, lib=lib)
    allowed = _allowed_from_ids(ids, B, T, S, Hq, Hkv, block)
    O_ref, lse_ref = _sdpa_reference(Q, K, V, allowed, 1.0 / np.sqrt(d))
    np.testing.assert_allclose(O, O_ref.reshape(B * T, Hq, d), rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse, lse_ref.reshape(B * T, Hq), rtol=0, atol=1e-10)
    # an explicit scale is honoured
    O3, lse3 = orc.attention(Q.reshape(B * T, Hq, d), K, V, ids, rows, T=T, block=block,
                             scale=0.37, lib=lib)
    O3_ref, lse3_ref = _sdpa_reference(Q, K, V, allowed, 0.37)
    np.testing.assert_allclose(O3, O3_ref.reshape(B * T, Hq, d), rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse3, lse3_ref.reshape(B * T, Hq), rtol=0, atol=1e-10)


def pin_closed_forms(lib):
    rng = np.random.default_rng(17)
    B, T, S, Hq, Hkv, d, d_idx, block, k = 1, 80, 120, 4, 2, 8, 4, 8, 4
    NB = -(-S // block)
    rows = _rows_all(B, T)
    # all-equal index scores: the tie-break alone decides -> {0..k-2} + {cb}
    q0 = np.zeros((B * T, Hkv, d_idx), np.float32)
    kk = _grid(rng, (B, S, d_idx))
    bs = orc.block_scores(q0, kk, rows, T=T, block=block, lib=lib)
    ids = orc.select_blocks(bs, rows, T=T, S=S, block=block, topk=k, lib=lib)
    for ri in range(B * T):
        cb = (S - T + ri) // block
        want = sorted(set(range(min(k - 1, cb))) | {cb})
        for g in range(Hkv):
            assert list(ids[ri, g, :len(want)]) == want
            assert np.all(ids[ri, g, len(want):] == -1)
            # only blocks with a causal token score finitely
            assert np.all(np.isfinite(bs[ri, g, :cb + 1])) and np.all(bs[ri, g, cb + 1:] == -np.inf)
    # constant values per (KV head, channel): output equals that constant
    Q = rng.standard_normal((B * T, Hq, d)).astype(np.float32)
    K = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
    c = rng.standard_normal((Hkv, d)).astype(np.float32)
    V = np.broadcast_to(c, (B, S, Hkv, d)).copy()
    O, lse = orc.attention(Q, K, V, ids, rows, T=T, block=block, lib=lib)
    R = Hq // Hkv
    for h in range(Hq):
        np.testing.assert_allclose(O[:, h, :], np.broadcast_to(c[h // R], (B * T, d)),
                                   rtol=0, atol=1e-12)
    # random values: output inside the per-channel hull of the attended rows,
    # and max_j s_j <= lse <= max_j s_j + log(#keys)
    V = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
    O, lse = orc.attention(Q, K, V, ids, rows, T=T, block=block, lib=lib)
    for ri in range(B * T):
        p = S - T + ri
        for h in range(Hq):
            g = h // R
            keys = [j for n in ids[ri, g] if n >= 0
                    for j in range(n * block, min((n + 1) * block, S)) if j <= p]
            vv = V[0, keys, g, :].astype(np.float64)
            assert np.all(O[ri, h] >= vv.min(0) - 1e-12) and np.all(O[ri, h] <= vv.max(0) + 1e-12)
            s = (K[0, keys, g, :].astype(np.float64) @ Q[ri, h].astype(np.float64)) / np.sqrt(d)
            assert s.max() - 1e-12 <= lse[ri, h] <= s.max() + np.log(len(keys)) + 1e-12
    # a query at position 0 attends exactly one key: O = V[0], lse = s_0
    T1, S1 = 4, 4
    Q1 = rng.standard_normal((T1, Hq, d)).astype(np.float32)
    K1 = rng.standard_normal((1, S1, Hkv, d)).astype(np.float32)
    V1 = rng.standard_normal((1, S1, Hkv, d)).astype(np.float32)
    ids1 = np.zeros((T1, Hkv, 1), np.int32)
    O1, lse1 = orc.attention(Q1, K1, V1, ids1, np.arange(T1), T=T1, block=block, lib=lib)
    for h in range(Hq):
        g = h // R
        np.testing.assert_allclose(O1[0, h], V1[0, 0, g], rtol=0, atol=1e-12)
        s0 = float(Q1[0, h].astype(np.float64) @ K1[0, 0, g].astype(np.float64)) / np.sqrt(d)
        np.testing.assert_allclose(lse1[0, h], s0, rtol=0, atol=1e-12)


def pin_permutation_invariance(lib):
    rng = np.random.default_rng(19)
    B, T, S, Hq, Hkv, d, block, k = 1, 64, 64, 4, 2, 8, 8, 4
    rows = _rows_all(B, T)
    Q = rng.standard_normal((B * T, Hq, d)).astype(np.float32)
    K = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
    q_idx = _grid(rng, (B * T, Hkv, 4))
    k_idx = _grid(rng, (B, S, 4))
    ids, O, lse = orc.forward(q_idx, k_idx, Q, K, V, rows, T=T, block=block, topk=k, lib=lib)
    perm = ids.copy()
    for ri in range(B * T):
        for g in range(Hkv):
            rng.shuffle(perm[ri, g])
    O2, lse2 = orc.attention(Q, K, V, perm, rows, T=T, block=block, lib=lib)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)


def pin_bf16_widening(lib):
    """The same grid values stored as bf16 and as fp32 give identical results
    (bf16 -> fp64 widening is exact)."""
    rng = np.random.default_rng(23)
    B, T, S, Hq, Hkv, d, d_idx, block, k = 1, 48, 48, 4, 2, 8, 8, 8, 3
    rows = _rows_all(B, T)
    q_idx = torch.from_numpy(_grid(rng, (B * T, Hkv, d_idx)))
    k_idx = torch.from_numpy(_grid(rng, (B, S, d_idx)))
    Q = torch.randn(B * T, Hq, d, generator=torch.Generator().manual_seed(3)).bfloat16()
    K = torch.randn(B, S, Hkv, d, generator=torch.Generator().manual_seed(4)).bfloat16()
    V = torch.randn(B, S, Hkv, d, generator=torch.Generator().manual_seed(5)).bfloat16()
    a = orc.forward(q_idx.bfloat16(), k_idx.bfloat16(), Q, K, V, rows, T=T, block=block,
                    topk=k, lib=lib, want_scores=True)
    b = orc.forward(q_idx, k_idx, Q.float(), K.float(), V.float(), rows, T=T, block=block,
                    topk=k, lib=lib, want_scores=True)
    for x, y in zip(a, b):
        assert np.array_equal(x, y), "bf16 and fp32 copies of the same values disagree"
    ma = orc.block_mass(Q, K, a[0], a[2], rows, T=T, block=block, lib=lib)
    mb = orc.block_mass(Q.float(), K.float(), b[0], b[2], rows, T=T, block=block, lib=lib)
    assert np.array_equal(ma, mb), "bf16 and fp32 copies give different block masses"


def _torch_block_mass(Q, K, allowed, scale, ids, block):
    """Head-averaged softmax mass of each kept slot's block from torch (fp64):
    softmax over the allowed tokens of the full score matrix, summed over the
    block's tokens, averaged over the group's heads.  [B*T, Hkv, topk]."""
    B, T, Hq, d = Q.shape
    S, Hkv = K.shape[1], K.shape[2]
    R = Hq // Hkv
    q = torch.from_numpy(Q.astype(np.float64)).permute(0, 2, 1, 3)           # B Hq T d
    k = torch.from_numpy(K.astype(np.float64)).permute(0, 2, 1, 3).repeat_interleave(R, dim=1)
    m = torch.from_numpy(allowed).permute(0, 2, 1, 3)                        # B Hq T S
    s = ((q @ k.transpose(-1, -2)) * scale).masked_fill(~m, float("-inf"))
    probs = torch.nan_to_num(torch.softmax(s, dim=-1)).numpy()               # B Hq T S
    tok_block = np.arange(S) // block
    out = np.zeros((B * T, Hkv, ids.shape[-1]))
    for b in range(B):
        for t in range(T):
            for g in range(Hkv):
                for i, n in enumerate(ids[b * T + t, g]):
                    if n >= 0:
                        out[b * T + t, g, i] = probs[b, g * R:(g + 1) * R, t][:, tok_block == n] \
                            .sum(axis=1).mean()
    return out


def pin_block_mass(lib):
    """The indexer's KL target (head-averaged block mass under the stored
    LSE) equals torch's masked softmax summed per block, for the dense limit
    and for sparse kept sets; it sums to 1 per row and group; with all
    scores equal it is the block's share of the attended tokens; with every
    head's LSE at -inf it is 0."""
    rng = np.random.default_rng(29)
    for B, T, S, Hq, Hkv, d, d_idx, block, k in [(1, 40, 40, 4, 2, 8, 4, 8, 5),
                                                (2, 24, 72, 6, 3, 16, 4, 8, 3),
                                                (1, 64, 64, 8, 2, 8, 4, 8, 2)]:
        NB = -(-S // block)
        Q = rng.standard_normal((B, T, Hq, d)).astype(np.float32)
        K = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
        V = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
        rows = _rows_all(B, T)
        Qr = Q.reshape(B * T, Hq, d)
        q_idx = _grid(rng, (B * T, Hkv, d_idx))
        k_idx = _grid(rng, (B, S, d_idx))
        for topk in (NB, k):                      # dense limit, then a sparse kept set
            ids, O, lse = orc.forward(q_idx, k_idx, Qr, K, V, rows, T=T, block=block,
                                      topk=topk, lib=lib)
            mass = orc.block_mass(Qr, K, ids, lse, rows, T=T, block=block, lib=lib)
            allowed = _allowed_from_ids(ids, B, T, S, Hq, Hkv, block)
            ref = _torch_block_mass(Q, K, allowed, 1.0 / np.sqrt(d), ids, block)
            np.testing.assert_allclose(mass, ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(mass.sum(-1), 1.0, rtol=0, atol=1e-12)
            assert np.all(mass[ids < 0] == 0.0)
        # all scores equal (K = 0): each kept block holds its share of the attended tokens
        K0 = np.zeros_like(K)
        ids, O, lse = orc.forward(q_idx, k_idx, Qr, K0, V, rows, T=T, block=block, topk=k,
                                  lib=lib)
        mass = orc.block_mass(Qr, K0, ids, lse, rows, T=T, block=block, lib=lib)
        for ri in range(B * T):
            p = S - T + ri % T
            for g in range(Hkv):
                kept = ids[ri, g]
                count = {n: min(p + 1, (n + 1) * block, S) - n * block for n in kept if n >= 0}
                total = sum(count.values())
                for i, n in enumerate(kept):
                    want = count[n] / total if n >= 0 else 0.0
                    assert abs(mass[ri, g, i] - want) < 1e-15, (ri, g, i)
        # no attended key anywhere (every LSE -inf): no mass
        none = orc.block_mass(Qr, K, ids, np.full_like(lse, -np.inf), rows, T=T, block=block,
                              lib=lib)
        assert np.all(none == 0.0)
    # a slot's mass is the head average of exp(LSE over that block alone - LSE over
    # the whole kept set), the single-block LSEs taken from the attention routine
    B, T, S, Hq, Hkv, d, d_idx, block, k = 1, 48, 96, 6, 2, 8, 4, 8, 4
    R = Hq // Hkv
    Q = rng.standard_normal((B * T, Hq, d)).astype(np.float32)
    K = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((B, S, Hkv, d)).astype(np.float32)
    rows = _rows_all(B, T)
    q_idx = _grid(rng, (B * T, Hkv, d_idx))
    k_idx = _grid(rng, (B, S, d_idx))
    ids, O, lse = orc.forward(q_idx, k_idx, Q, K, V, rows, T=T, block=block, topk=k, lib=lib)
    mass = orc.block_mass(Q, K, ids, lse, rows, T=T, block=block, lib=lib)
    for i in range(k):
        one = np.full_like(ids, -1)
        one[..., 0] = ids[..., i]
        _, lse_i = orc.attention(Q, K, V, one, rows, T=T, block=block, lib=lib)
        want = np.exp(lse_i - lse).reshape(B * T, Hkv, R).mean(-1)
        want[ids[..., i] < 0] = 0.0
        np.testing.assert_allclose(mass[..., i], want, rtol=1e-12, atol=1e-15)


def make_paged(rng, dense_rows_list, page_size, spare_pages=3):
    """Scatter each sequence's rows (a list of [L_b, ...] arrays) over pages
    in a random order.  Returns (cache [num_pages, page_size, ...],
    block_table [B, max_pages]); unused table entries hold a valid page id."""
    B = len(dense_rows_list)
    n_pages = [-(-len(x) // page_size) for x in dense_rows_list]
    max_pages = max(n_pages) + 1
    num_pages = sum(n_pages) + spare_pages
    order = rng.permutation(num_pages)
    tail = dense_rows_list[0].shape[1:]
    cache = rng.standard_normal((num_pages, page_size) + tail).astype(np.float32)
    table = np.zeros((B, max_pages), dtype=np.int32)
    k = 0
    for b, x in enumerate(dense_rows_list):
        for i in range(n_pages[b]):
            pg = int(order[k])
            k += 1
            table[b, i] = pg
            rows = x[i * page_size:(i + 1) * page_size]
            cache[pg, :len(rows)] = rows
    return cache, table


def pin_paged_addressing(lib):
    """The paged forward equals, sequence by sequence, the method on that
    sequence's keys laid out densely, computed without the oracle: block
    scores from the full score matrix, kept sets by counting, attention by
    SDPA with the kept-block mask.  Lengths not a multiple of the block,
    pages scattered in random order, page sizes below and above the block."""
    rng = np.random.default_rng(23)
    T, Hq, Hkv, d, d_idx, block, k, S = 2, 4, 2, 16, 8, 16, 4, 160
    for page_size, lens in [(8, [160, 123, 40]), (24, [97, 160, 2])]:
        B = len(lens)
        q_idx = _grid(rng, (B, T, Hkv, d_idx))
        Q = rng.standard_normal((B, T, Hq, d)).astype(np.float32)
        kd = [_grid(rng, (L, d_idx)) for L in lens]
        Kd = [rng.standard_normal((L, Hkv, d)).astype(np.float32) for L in lens]
        Vd = [rng.standard_normal((L, Hkv, d)).astype(np.float32) for L in lens]
        kc, table = make_paged(rng, kd, page_size)
        # one table for all three caches: K and V on the index keys' pages
        Kc = np.zeros((kc.shape[0], page_size, Hkv, d), np.float32)
        Vc = np.zeros((kc.shape[0], page_size, Hkv, d), np.float32)
        for b, L in enumerate(lens):
            for j in range(L):
                pg, off = table[b, j // page_size], j % page_size
                Kc[pg, off], Vc[pg, off] = Kd[b][j], Vd[b][j]
        ids, O, lse = orc.forward_paged(q_idx, kc, Q, Kc, Vc, np.array(lens), table, S=S,
                                        block=block, topk=k, lib=lib)
        for b, L in enumerate(lens):
            bs = brute_block_scores(q_idx[b:b + 1], kd[b][None], T, block)[0]     # [T, G, NB]
            for t in range(T):
                cb = (L - T + t) // block
                for g in range(Hkv):
                    want = sorted(brute_kept_sets(bs[t, g], cb, k))
                    got = [int(x) for x in ids[b, t, g] if x >= 0]
                    assert got == want, (page_size, b, t, g, got, want)
                    assert all(x == -1 for x in ids[b, t, g, len(want):])
            allowed = _allowed_from_ids(ids[b].reshape(T, Hkv, k), 1, T, L, Hq, Hkv, block)
            O_ref, lse_ref = _sdpa_reference(Q[b:b + 1], Kd[b][None], Vd[b][None], allowed,
                                             1.0 / np.sqrt(d))
            np.testing.assert_allclose(O[b], O_ref[0], rtol=0, atol=1e-10)
            np.testing.assert_allclose(lse[b], lse_ref[0], rtol=0, atol=1e-10)


def brute_hierarchical(q_idx, k_idx, T, block, k, kc):
    """Coarse-to-fine kept sets [B, T, G] of python sets, by numpy and by
    counting: block means by reshape, coarse scores by matmul, candidates
    = earlier blocks with fewer than kc - 1 better coarse scores, kept = the
    current block and the candidates with fewer than k - 1 better fine
    (exact max-pooled) scores among the candidates."""
    B, _, G, d_idx = q_idx.shape
    S = k_idx.shape[1]
    NB = S // block
    mean = k_idx.astype(np.float64).reshape(B, NB, block, d_idx).mean(axis=2)   # [B, NB, d]
    coarse = np.einsum("btgi,bni->btgn", q_idx.astype(np.float64), mean)
    fine = brute_block_scores(q_idx, k_idx, T, block)
    out = np.empty((B, T, G), dtype=object)
    for b in range(B):
        for t in range(T):
            cb = (S - T + t) // block
            for g in range(G):
                c = coarse[b, t, g]
                cands = [n for n in range(cb)
                         if sum(1 for m in range(cb)
                                if c[m] > c[n] or (c[m] == c[n] and m < n)) < kc - 1]
                f = fine[b, t, g]
                kept = {n for n in cands
                        if sum(1 for m in cands
                               if f[m] > f[n] or (f[m] == f[n] and m < n)) < k - 1}
                out[b, t, g] = kept | {cb}
    return out


def pin_hierarchical_selection(lib):
    """The coarse-to-fine selection equals the brute-force count on tiny
    inputs (several candidate counts), and with every earlier block a
    candidate it is the exact selection."""
    rng = np.random.default_rng(29)
    for B, T, S, G, d_idx, block, k, kcs in [(1, 40, 160, 2, 8, 8, 3, (3, 5, 9)),
                                            (2, 24, 96, 1, 4, 16, 2, (2, 4))]:
        q_idx = _grid(rng, (B, T, G, d_idx))
        k_idx = _grid(rng, (B, S, d_idx))
        rows = _rows_all(B, T)
        NB = S // block
        for kc in kcs + (NB + 1,):
            ids = orc.select_hierarchical(q_idx.reshape(B * T, G, d_idx), k_idx, rows, T=T,
                                          block=block, topk=k, kc=kc, lib=lib)
            want = brute_hierarchical(q_idx, k_idx, T, block, k, kc)
            for r in range(B * T):
                for g in range(G):
                    got = ids[r, g]
                    kept = sorted(want[r // T, r % T, g])
                    assert list(got[:len(kept)]) == kept, (kc, r, g, got, kept)
                    assert all(x == -1 for x in got[len(kept):])
        # every earlier block a candidate: the exact selection
        exact = orc.select_blocks(orc.block_scores(q_idx.reshape(B * T, G, d_idx), k_idx, rows,
                                                   T=T, block=block, lib=lib),
                                  rows, T=T, S=S, block=block, topk=k, lib=lib)
        full = orc.select_hierarchical(q_idx.reshape(B * T, G, d_idx), k_idx, rows, T=T,
                                       block=block, topk=k, kc=NB, lib=lib)
        assert np.array_equal(full, exact)


ALL_PINS = [pin_brute_force_selection, pin_dense_limit, pin_masked_attention,
            pin_closed_forms, pin_permutation_invariance, pin_bf16_widening, pin_block_mass,
            pin_paged_addressing, pin_hierarchical_selection]
