"""The oracle against the numbers the pages print.

"MiniMax Sparse Attention -- paper by Lai et al. (2026)", Key points,
"Benchmark configuration": B_k = 128 and k = 16 give 2,048 attended tokens
per query, with 64 query heads, 4 KV heads and head dimension 128.  Under
the reading that the forced current block is one of the k, a query whose
current block is full and has at least 15 earlier blocks attends exactly
k * B_k = 2048 tokens.  The count is read off the oracle's LSE: with all
keys zero every attended score is 0, so LSE = log(#attended tokens).
"""
import json
import math
import os

import numpy as np

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "msa_benchmark_configuration.json")


def test_attended_tokens_per_query():
    cfg = json.load(open(GOLDEN))
    Bk, k, Hq, Hkv, d = cfg["block"], cfg["topk"], cfg["query_heads"], cfg["kv_heads"], cfg["head_dim"]
    S = T = Bk * 20
    rng = np.random.default_rng(0)
    positions = [Bk * 16 - 1, Bk * 17 - 1, Bk * 20 - 1,   # full current block, cb >= 15
                 Bk * 16,                                 # first token of block 16
                 Bk * 3 + 5]                              # fewer than k causal blocks
    rows = np.array(positions, dtype=np.int64)
    q_idx = (rng.integers(-4, 5, size=(len(rows), Hkv, 8)) / 4).astype(np.float32)
    k_idx = (rng.integers(-4, 5, size=(1, S, 8)) / 4).astype(np.float32)
    Q = rng.standard_normal((len(rows), Hq, d)).astype(np.float32)
    K = np.zeros((1, S, Hkv, d), np.float32)
    V = rng.standard_normal((1, S, Hkv, d)).astype(np.float32)
    ids, O, lse = orc.forward(q_idx, k_idx, Q, K, V, rows, T=T, block=Bk, topk=k)
    counts = np.exp(lse)
    expect = {Bk * 16 - 1: cfg["attended_tokens_per_query"],
              Bk * 17 - 1: cfg["attended_tokens_per_query"],
              Bk * 20 - 1: cfg["attended_tokens_per_query"],
              Bk * 16: (k - 1) * Bk + 1,
              Bk * 3 + 5: Bk * 3 + 6}
    for ri, p in enumerate(positions):
        assert np.all(ids[ri] >= -1)
        np.testing.assert_allclose(counts[ri], expect[p], rtol=1e-12)
        n_kept = (ids[ri] >= 0).sum(axis=-1)
        assert np.all(n_kept == min(k, p // Bk + 1))
    assert math.isclose(k * Bk, cfg["attended_tokens_per_query"])
