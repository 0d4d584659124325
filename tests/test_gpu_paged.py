"""msa_decode_paged: decode steps over a paged KV cache with per-sequence
lengths, against the oracle's paged forward (ids bit-exact; O, LSE within
the bf16 tolerance of tests/parity.py).

Lengths mix full, one short of full, not a multiple of the block, one
block, one token past a block, and the minimum (T); pages are scattered in
random order, with page sizes below, equal to and above the block.  With
contiguous pages and every length at capacity the call is bitwise
msa_forward on the dense cache.  Bad lengths and page ids are skipped and
reported without touching the other sequences."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def _msa():
    import block_sparse_long_03_b200 as msa
    return msa


def _paged_inputs(w, lens, page_size, seed):
    """Dense synthetic inputs of workload w, with each sequence's index keys,
    K and V scattered over pages in a random order (one table for all three
    caches).  Returns (inp, k_idx_cache, K_cache, V_cache, table, num_pages)."""
    from block_sparse_long_03_b200 import synthetic
    inp = synthetic.make_inputs(w, seed, device="cpu")
    g = torch.Generator().manual_seed(seed + 100)
    n_pages = [-(-L // page_size) for L in lens]
    max_pages = -(-w.S // page_size)
    num_pages = sum(n_pages) + 5
    order = torch.randperm(num_pages, generator=g)
    table = torch.full((w.B, max_pages), -1, dtype=torch.int32)
    kc = torch.zeros((num_pages, page_size, w.d_idx), dtype=w.dtype)
    Kc = torch.zeros((num_pages, page_size, w.Hkv, w.d), dtype=w.dtype)
    Vc = torch.zeros((num_pages, page_size, w.Hkv, w.d), dtype=w.dtype)
    k = 0
    for b, L in enumerate(lens):
        for i in range(n_pages[b]):
            pg = int(order[k])
            k += 1
            table[b, i] = pg
            lo, hi = i * page_size, min(w.S, (i + 1) * page_size)
            kc[pg, :hi - lo] = inp.k_idx[b, lo:hi]
            Kc[pg, :hi - lo] = inp.K[b, lo:hi]
            Vc[pg, :hi - lo] = inp.V[b, lo:hi]
    return inp, kc, Kc, Vc, table, num_pages


def _run(w, lens, page_size, seed, table_edit=None, lens_gpu=None):
    msa = _msa()
    inp, kc, Kc, Vc, table, num_pages = _paged_inputs(w, lens, page_size, seed)
    if table_edit is not None:
        table_edit(table)
    lg = torch.tensor(lens if lens_gpu is None else lens_gpu, dtype=torch.int32).cuda()
    O, lse, ids, ws = msa.decode_paged(inp.q_idx.cuda(), kc.cuda(), inp.Q.cuda(), Kc.cuda(),
                                       Vc.cuda(), lg, table.cuda(), S=w.S, block=w.block,
                                       topk=w.topk)
    torch.cuda.synchronize()
    return inp, kc, Kc, Vc, table, O, lse, ids, ws


CASES = [
    # (name, workload kwargs, lengths, page size)
    ("page16_block64", dict(B=6, T=1, S=4096, Hq=32, Hkv=8, block=64, topk=8),
     [4096, 4095, 1000, 64, 65, 1], 16),
    ("page64_block64", dict(B=5, T=1, S=8192, Hq=32, Hkv=8, block=64, topk=32),
     [8192, 5000, 2049, 700, 3000], 64),
    ("page48_block128_T4", dict(B=4, T=4, S=4096, Hq=16, Hkv=2, block=128, topk=6),
     [4096, 1234, 4, 129], 48),
    ("page256_R16", dict(B=3, T=1, S=4096, Hq=32, Hkv=2, block=128, topk=6),
     [3333, 4096, 200], 256),
]


@pytest.mark.parametrize("name,kw,lens,page_size", CASES, ids=[c[0] for c in CASES])
def test_paged_decode_matches_oracle(name, kw, lens, page_size):
    from block_sparse_long_03_b200 import synthetic
    w = synthetic.Workload(name, d=128, d_idx=64, dtype=torch.bfloat16, **kw)
    inp, kc, Kc, Vc, table, O, lse, ids, ws = _run(w, lens, page_size, seed=3)
    msa = _msa()
    assert msa.msa_get_device_error(ws) == 0
    ids_ref, O_ref, lse_ref = orc.forward_paged(inp.q_idx, kc, inp.Q, Kc, Vc, np.array(lens),
                                                table.numpy(), S=w.S, block=w.block,
                                                topk=w.topk)
    parity.assert_ids_equal(ids.cpu().numpy().reshape(-1, w.G, w.topk),
                            ids_ref.reshape(-1, w.G, w.topk), name)
    parity.assert_close(O.float().cpu().numpy().reshape(-1, w.Hq, w.d),
                        lse.cpu().numpy().reshape(-1, w.Hq), O_ref.reshape(-1, w.Hq, w.d),
                        lse_ref.reshape(-1, w.Hq), w.dtype, name)


def test_contiguous_pages_equal_dense_forward():
    """Pages laid out in order with every sequence at capacity: the paged
    call reads exactly the dense cache, and its outputs are bitwise those of
    msa_forward on it."""
    msa = _msa()
    from block_sparse_long_03_b200 import synthetic
    w = synthetic.Workload("paged_dense", B=4, T=1, S=4096, Hq=32, Hkv=8, d=128, d_idx=64,
                           block=64, topk=16, dtype=torch.bfloat16)
    inp = synthetic.make_inputs(w, 9, device="cuda")
    page_size = 128
    per = w.S // page_size
    table = torch.arange(w.B * per, dtype=torch.int32, device="cuda").view(w.B, per)
    lens = torch.full((w.B,), w.S, dtype=torch.int32, device="cuda")
    O, lse, ids, ws = msa.decode_paged(
        inp.q_idx, inp.k_idx.view(-1, page_size, w.d_idx), inp.Q,
        inp.K.view(-1, page_size, w.Hkv, w.d), inp.V.view(-1, page_size, w.Hkv, w.d), lens,
        table, S=w.S, block=w.block, topk=w.topk)
    O2, lse2, ids2, ws2 = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                      topk=w.topk)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    assert torch.equal(ids, ids2)
    assert torch.equal(lse, lse2)
    assert torch.equal(O.view(torch.int16), O2.view(torch.int16))


def test_bad_lengths_and_pages_are_skipped():
    """A page id past the pool, a length above capacity and a length below T:
    those sequences get ids -1, O = 0 and lse = -inf, the error word says
    MSA_ERR_BAD_PAGE_TABLE, and the other sequences match the oracle."""
    msa = _msa()
    from block_sparse_long_03_b200 import synthetic
    w = synthetic.Workload("paged_bad", B=5, T=1, S=2048, Hq=16, Hkv=4, d=128, d_idx=64,
                           block=64, topk=8, dtype=torch.bfloat16)
    lens = [2048, 1500, 900, 2000, 1777]

    def plant(table):
        table[1, 3] = 1 << 20                         # page id past the pool

    lens_gpu = list(lens)
    lens_gpu[2] = w.S + 1                             # above capacity
    lens_gpu[3] = 0                                   # below T
    inp, kc, Kc, Vc, table, O, lse, ids, ws = _run(w, lens, 32, seed=5, table_edit=plant,
                                                   lens_gpu=lens_gpu)
    assert msa.msa_get_device_error(ws) == 7
    for b in (1, 2, 3):
        assert bool((ids[b] == -1).all())
        assert bool((O[b] == 0).all())
        assert bool(torch.isinf(lse[b]).all() and (lse[b] < 0).all())
    good = [0, 4]
    sel = torch.tensor(good)
    t_good = table[sel]
    ids_ref, O_ref, lse_ref = orc.forward_paged(
        inp.q_idx[sel], kc, inp.Q[sel], Kc, Vc, np.array([lens[b] for b in good]),
        t_good.numpy(), S=w.S, block=w.block, topk=w.topk)
    parity.assert_ids_equal(ids[sel].cpu().numpy().reshape(-1, w.G, w.topk),
                            ids_ref.reshape(-1, w.G, w.topk), "bad pages")
    parity.assert_close(O[sel].float().cpu().numpy().reshape(-1, w.Hq, w.d),
                        lse[sel].cpu().numpy().reshape(-1, w.Hq), O_ref.reshape(-1, w.Hq, w.d),
                        lse_ref.reshape(-1, w.Hq), w.dtype, "bad pages")
