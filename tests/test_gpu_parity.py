"""CUDA library vs the fp64 oracle, element by element, on small workloads
that span several tiles and ragged tails (the oracle runs on every row).

Tolerances live in tests/parity.py: ids and block scores bit-exact; O
max-abs 2e-2 / mean-abs 2e-3 (bf16), 1e-4 (fp32); LSE 2e-3 / 1e-5."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def _msa():
    import block_sparse_long_03_b200 as msa
    return msa


def _synth():
    from block_sparse_long_03_b200 import synthetic
    return synthetic


def _case(name):
    W = _synth().Workload
    bf = torch.bfloat16
    cases = {
        "tiny_fp32_prefill": _synth().WORKLOADS["tiny_fp32_prefill"],
        "bf16_prefill_2x1024": W("bf16_prefill_2x1024", B=2, T=1024, S=1024, Hq=8, Hkv=2, d=128,
                                 d_idx=64, block=128, topk=4, dtype=bf, hot_blocks_per_group=2),
        "bf16_chunk_ragged": W("bf16_chunk_ragged", B=1, T=200, S=1024, Hq=16, Hkv=2, d=128,
                               d_idx=64, block=64, topk=6, dtype=bf),
        "bf16_decode_small": W("bf16_decode_small", B=8, T=1, S=2048, Hq=32, Hkv=8, d=128,
                               d_idx=64, block=64, topk=8, dtype=bf),
        "bf16_d64_mha": W("bf16_d64_mha", B=1, T=512, S=512, Hq=4, Hkv=4, d=64, d_idx=32,
                          block=64, topk=3, dtype=bf),
        "bf16_dense_limit": W("bf16_dense_limit", B=1, T=512, S=512, Hq=8, Hkv=1, d=128,
                              d_idx=16, block=64, topk=8, dtype=bf),
        "bf16_topk1": W("bf16_topk1", B=1, T=256, S=256, Hq=4, Hkv=2, d=128, d_idx=64,
                        block=64, topk=1, dtype=bf),
        "fp32_gqa8": W("fp32_gqa8", B=1, T=384, S=512, Hq=16, Hkv=2, d=128, d_idx=64,
                       block=128, topk=3, dtype=torch.float32),
        # tensor-core prefill path across group sizes, index widths and batching
        "bf16_prefill_R16": W("bf16_prefill_R16", B=1, T=1024, S=1024, Hq=32, Hkv=2, d=128,
                              d_idx=64, block=128, topk=4, dtype=bf, hot_blocks_per_group=1),
        "bf16_prefill_R1_didx128": W("bf16_prefill_R1_didx128", B=1, T=512, S=512, Hq=4, Hkv=4,
                                     d=128, d_idx=128, block=64, topk=5, dtype=bf),
        "bf16_prefill_B2_chunk": W("bf16_prefill_B2_chunk", B=2, T=300, S=1024, Hq=8, Hkv=4,
                                   d=128, d_idx=64, block=128, topk=3, dtype=bf),
        # decode path: block 128, several query tokens, 64 kept blocks (two slot passes)
        "bf16_decode_block128": W("bf16_decode_block128", B=3, T=1, S=4096, Hq=16, Hkv=2, d=128,
                                  d_idx=64, block=128, topk=6, dtype=bf),
        "bf16_decode_T4": W("bf16_decode_T4", B=2, T=4, S=2048, Hq=8, Hkv=2, d=128, d_idx=64,
                            block=64, topk=4, dtype=bf),
        "bf16_decode_topk64": W("bf16_decode_topk64", B=2, T=1, S=8192, Hq=32, Hkv=4, d=128,
                                d_idx=64, block=64, topk=64, dtype=bf),
        # an odd number of 64-key blocks: the last 128-key index tile holds one block
        "bf16_prefill_odd_blocks": W("bf16_prefill_odd_blocks", B=2, T=700, S=1088, Hq=8, Hkv=2,
                                     d=128, d_idx=64, block=64, topk=5, dtype=bf),
        # decode with 16 heads per group: two CTAs of 8 heads per kept block
        "bf16_decode_R16": W("bf16_decode_R16", B=3, T=1, S=4096, Hq=32, Hkv=2, d=128,
                             d_idx=64, block=128, topk=6, dtype=bf),
        # more than 2048 candidate blocks per row: the CTA-per-row Top-k
        "bf16_chunk_many_blocks": W("bf16_chunk_many_blocks", B=1, T=64, S=139264, Hq=8, Hkv=2,
                                    d=128, d_idx=64, block=64, topk=9, dtype=bf),
        # more than 64 kept blocks (batched merge), 16 heads per group with 64
        # kept blocks, head dimension 64 on the tensor-core path (TMA Q boxes
        # and the cp.async Q gather), and T = 1 with d = 64 (tensor-core path)
        "bf16_prefill_topk128": W("bf16_prefill_topk128", B=1, T=512, S=16384, Hq=16, Hkv=2,
                                  d=128, d_idx=64, block=64, topk=128, dtype=bf),
        "bf16_prefill_R16_topk64": W("bf16_prefill_R16_topk64", B=1, T=384, S=8192, Hq=32,
                                     Hkv=2, d=128, d_idx=64, block=64, topk=64, dtype=bf),
        "bf16_decode_topk128": W("bf16_decode_topk128", B=2, T=1, S=16384, Hq=16, Hkv=4, d=128,
                                 d_idx=64, block=64, topk=128, dtype=bf),
        "bf16_d64_R8": W("bf16_d64_R8", B=1, T=768, S=1024, Hq=16, Hkv=2, d=64, d_idx=64,
                         block=128, topk=4, dtype=bf, hot_blocks_per_group=1),
        "bf16_decode_d64": W("bf16_decode_d64", B=4, T=1, S=2048, Hq=8, Hkv=2, d=64, d_idx=64,
                             block=64, topk=8, dtype=bf),
    }
    return cases[name]


CASES = ["tiny_fp32_prefill", "bf16_prefill_2x1024", "bf16_chunk_ragged", "bf16_decode_small",
         "bf16_d64_mha", "bf16_dense_limit", "bf16_topk1", "fp32_gqa8", "bf16_prefill_R16",
         "bf16_prefill_R1_didx128", "bf16_prefill_B2_chunk", "bf16_decode_block128",
         "bf16_decode_T4", "bf16_decode_topk64", "bf16_prefill_odd_blocks",
         "bf16_chunk_many_blocks", "bf16_decode_R16", "bf16_prefill_topk128",
         "bf16_prefill_R16_topk64", "bf16_decode_topk128", "bf16_d64_R8", "bf16_decode_d64"]


def _inputs(w, seed=0):
    inp = _synth().make_inputs(w, seed, device="cpu")
    for f in ("q_idx", "k_idx", "Q", "K", "V"):
        setattr(inp, f, getattr(inp, f).cuda())
    return inp


@pytest.mark.parametrize("name", CASES)
def test_forward_matches_oracle(name):
    msa = _msa()
    w = _case(name)
    inp = _inputs(w)
    O, lse, ids, ws = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                  topk=w.topk)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    rows = list(range(w.B * w.T))
    ref = parity.oracle_rows(inp, w, rows)
    parity.assert_ids_equal(parity.gather_rows(ids, rows, w.T), ref["ids"], name)
    parity.assert_close(parity.gather_rows(O, rows, w.T), parity.gather_rows(lse, rows, w.T),
                        ref["O"], ref["lse"], w.dtype, name)


@pytest.mark.parametrize("name", ["tiny_fp32_prefill", "bf16_chunk_ragged", "bf16_decode_small",
                                  "bf16_prefill_odd_blocks", "bf16_prefill_B2_chunk",
                                  "bf16_prefill_R1_didx128"])
def test_index_scores_and_topk_calls(name):
    """The two index-branch calls on their own: block scores bit-exact (the
    -inf of every non-causal block included: odd block counts, T < S and
    two sequences exercise the fill's unaligned head and tail), and Top-k
    run on the ORACLE's block scores gives the oracle's ids."""
    msa = _msa()
    w = _case(name)
    inp = _inputs(w, seed=3)
    bs = msa.index_block_scores(inp.q_idx, inp.k_idx, block=w.block)
    rows = list(range(w.B * w.T))
    ref = parity.oracle_rows(inp, w, rows, want_scores=True)
    got = parity.gather_rows(bs, rows, w.T)
    parity.assert_bits_equal(got, ref["bs"], name)
    ref_bs = torch.from_numpy(ref["bs"].astype(np.float32)).reshape(w.B, w.T, w.G, w.NB).cuda()
    ids = msa.topk_blocks(ref_bs, S=w.S, block=w.block, topk=w.topk)
    parity.assert_ids_equal(parity.gather_rows(ids, rows, w.T), ref["ids"], name)


def test_topk_heavy_ties_and_closed_form():
    """All index scores equal: the tie-break alone decides, so each row keeps
    blocks {0..k-2} and its current block."""
    msa = _msa()
    B, T, S, G, block, k = 1, 700, 1024, 3, 64, 5
    NB = S // block
    bs = torch.zeros((B, T, G, NB), dtype=torch.float32, device="cuda")
    ids = msa.topk_blocks(bs, S=S, block=block, topk=k).cpu().numpy()
    for t in range(T):
        cb = (S - T + t) // block
        want = sorted(set(range(min(k - 1, cb))) | {cb})
        for g in range(G):
            assert list(ids[0, t, g, :len(want)]) == want
            assert np.all(ids[0, t, g, len(want):] == -1)


@pytest.mark.parametrize("name", ["bf16_chunk_ragged", "bf16_decode_small", "bf16_decode_T4",
                                  "bf16_decode_R16"])
def test_sparse_attn_permuted_and_bad_ids(name):
    """Caller ids in any order give the same result; ids out of range or
    repeated are skipped and reported through the device error word (the
    tensor-core prefill path and the decode path)."""
    msa = _msa()
    w = _case(name)
    inp = _inputs(w, seed=5)
    O, lse, ids, ws = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                  topk=w.topk)
    perm = ids.flip(-1).contiguous()
    O2, lse2, ws2 = msa.sparse_attn_fwd(inp.Q, inp.K, inp.V, perm, block=w.block)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws2) == 0
    tol = parity.TOL[w.dtype]
    assert (O2.float() - O.float()).abs().max().item() <= tol["o_max"]
    assert (lse2 - lse).abs().max().item() <= tol["lse_max"]
    # plant an out-of-range id and a repeat in every row's empty or first slot
    bad = ids.clone()
    bad[..., -1] = w.NB + 7
    bad[..., 0] = bad[..., 1]
    O3, lse3, ws3 = msa.sparse_attn_fwd(inp.Q, inp.K, inp.V, bad, block=w.block)
    assert msa.msa_get_device_error(ws3) == 6
    rows = list(range(0, w.B * w.T, 7))
    ref = parity.oracle_rows(inp, w, rows, ids=_dedup_valid(bad, w.NB))
    parity.assert_close(parity.gather_rows(O3, rows, w.T), parity.gather_rows(lse3, rows, w.T),
                        ref["O"], ref["lse"], w.dtype, "bad ids")


def _dedup_valid(ids, NB):
    """What the library must attend to: valid ids, each once."""
    out = ids.clone().cpu()
    flat = out.reshape(-1, out.shape[-1])
    for r in range(flat.shape[0]):
        seen = set()
        for i in range(flat.shape[1]):
            n = int(flat[r, i])
            if n < 0 or n >= NB or n in seen:
                flat[r, i] = -1
            else:
                seen.add(n)
    return out
