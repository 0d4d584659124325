"""How msa_forward and msa_forward_host cut the work into query pieces
(msa_query_pieces; host logic, no GPU): pieces of a sequence cover its
queries in order without gaps, every piece but the last of a sequence ends
where T - end is a multiple of the block (so its keys S' = S - T + end are
whole blocks), no piece is shorter than 128 queries, the forward's pieces
hold at most 1 GiB of block scores (plus the at most 127 queries a merged
short piece adds), and shapes that fit run whole."""
import pytest
import torch


def _p(**kw):
    from block_sparse_long_03_b200 import make_params
    base = dict(B=1, T=131072, S=131072, Hq=64, Hkv=8, d=128, d_idx=64, block=128, topk=32,
                dtype=torch.bfloat16)
    base.update(kw)
    return make_params(**base), base


def _check_cover(pieces, T, B, block):
    seqs = sorted({s for s, _, _ in pieces})
    if seqs == [-1]:
        assert pieces == [(-1, 0, T)]
        return
    assert seqs == list(range(B))
    for b in range(B):
        mine = [(t0, t1) for s, t0, t1 in pieces if s == b]
        assert mine[0][0] == 0 and mine[-1][1] == T
        for (a0, a1), (b0, _) in zip(mine, mine[1:]):
            assert a1 == b0, "gap or overlap"
        for t0, t1 in mine:
            assert t1 - t0 >= 128
            assert (T - t1) % block == 0


SHAPES = [dict(), dict(T=1 << 20, S=1 << 20, Hkv=4, topk=16),
          dict(B=2, T=147456, S=147456, Hq=8, Hkv=8, topk=8),
          dict(T=8232, S=8320, Hq=8, Hkv=2, block=64, topk=6),
          dict(T=5696, S=5696, Hq=8, Hkv=1, block=64, topk=6),
          dict(B=2, T=10240, S=10240, Hq=16, Hkv=2, topk=8),
          dict(B=64, T=1, S=131072, Hq=32, block=64),
          dict(T=200, S=1024, Hq=16, Hkv=2, block=64, topk=6)]


@pytest.mark.parametrize("kw", SHAPES)
def test_pieces_cover_in_block_steps(kw):
    import block_sparse_long_03_b200 as msa
    p, sh = _p(**kw)
    for which in (msa.MSA_WS_FORWARD, msa.MSA_WS_FORWARD_HOST):
        pieces = msa.msa_query_pieces(p, which)
        assert pieces, which
        _check_cover(pieces, sh["T"], sh["B"], sh["block"])


@pytest.mark.parametrize("kw", SHAPES)
def test_forward_pieces_bound_the_scores(kw):
    import block_sparse_long_03_b200 as msa
    p, sh = _p(**kw)
    NB = sh["S"] // sh["block"]
    full = sh["B"] * sh["T"] * sh["Hkv"] * NB * 4
    pieces = msa.msa_query_pieces(p, msa.MSA_WS_FORWARD)
    if full <= 4 << 30:
        assert pieces == [(-1, 0, sh["T"])]               # the whole array fits: one call
    else:
        for _, t0, t1 in pieces:
            assert (t1 - t0 - 127) * sh["Hkv"] * NB * 4 <= 1 << 30


def test_known_plans():
    import block_sparse_long_03_b200 as msa
    p, _ = _p()                                           # 128K: 4 GiB of scores, whole
    assert msa.msa_query_pieces(p, msa.MSA_WS_FORWARD) == [(-1, 0, 131072)]
    host = msa.msa_query_pieces(p, msa.MSA_WS_FORWARD_HOST)
    sizes = [t1 - t0 for _, t0, t1 in host]
    assert len(host) == 18 and sizes[0] == 896 and sizes[-1] == 1920
    assert set(sizes[1:-2]) == {8064}                     # one attention pass each
    p, _ = _p(T=1 << 20, S=1 << 20, Hkv=4, topk=16)       # the pages' 1M shape
    fwd = msa.msa_query_pieces(p, msa.MSA_WS_FORWARD)
    assert len(fwd) == 128 and all(t1 - t0 == 8192 for _, t0, t1 in fwd)
    p, _ = _p(B=64, T=1, S=131072, Hq=32, block=64)       # decode runs whole
    assert msa.msa_query_pieces(p, msa.MSA_WS_FORWARD_HOST) == [(-1, 0, 1)]


def test_query_pieces_rejects():
    import ctypes
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import binding
    p, _ = _p(T=0)
    assert binding.lib.msa_query_pieces(ctypes.byref(p), msa.MSA_WS_FORWARD, None, 0) == 0
    p, _ = _p()
    assert binding.lib.msa_query_pieces(ctypes.byref(p), 7, None, 0) == 0
    assert binding.lib.msa_query_pieces(ctypes.byref(p), msa.MSA_WS_FORWARD, None, 4) == -1


def test_workspace_stays_bounded_for_long_prefill():
    """msa_forward's workspace holds one piece's scores once the whole array
    passes 4 GiB (128 GiB at the pages' 1M shape), and the host call's buffer
    holds at least every tensor it copies plus that scratch."""
    import block_sparse_long_03_b200 as msa
    p, sh = _p(T=1 << 20, S=1 << 20, Hkv=4, topk=16)
    full_scores = sh["T"] * sh["Hkv"] * (sh["S"] // sh["block"]) * 4
    ws = msa.msa_workspace_size(p, msa.MSA_WS_FORWARD)
    assert full_scores == 128 << 30
    assert ws < 8 << 30                                   # partial budget + one piece of scores
    host = msa.msa_workspace_size(p, msa.MSA_WS_FORWARD_HOST)
    T, S, Hq, Hkv, d, d_idx = sh["T"], sh["S"], sh["Hq"], sh["Hkv"], sh["d"], sh["d_idx"]
    tensors = 2 * (T * Hkv * d_idx + S * d_idx + 2 * T * Hq * d + 2 * S * Hkv * d) + 4 * T * Hq
    assert host >= tensors
    p, _ = _p()                                           # 128K: the whole array, 4 GiB
    assert msa.msa_workspace_size(p, msa.MSA_WS_FORWARD) >= 4 << 30
