"""msa_forward_host (page-locked host buffers, copies overlapped with the
kernels) against msa_forward on the same inputs: O, lse and ids bitwise equal.

Every query row's arithmetic is the same whichever call or chunk it runs in
(index scores and Top-k run over all rows at once; the attention of a row
depends only on its own kept blocks, and its partials are combined in slot
order), so the host call must reproduce msa_forward exactly.  Shapes cover
sequences split into query chunks (several chunks, two sequences, T < S with
T not a multiple of the block, a piece under 128 queries merged into the
next, one KV group) and shapes that run whole (decode, fp32, short prefill);
the chunked case is also checked against the oracle on sampled rows and both
sides of every chunk boundary, and the full 128K prefill in the configuration
the end-to-end benchmark times."""
import pytest
import torch

from tests import parity

pytestmark = pytest.mark.gpu


def _synth():
    from block_sparse_long_03_b200 import synthetic
    return synthetic


def _case(name):
    W = _synth().Workload
    bf = torch.bfloat16
    return {
        # pieces [0, 512), [512, 4608), [4608, 8704), [8704, 9216), [9216, 10240)
        # of each of two sequences
        "chunked_B2": W("chunked_B2", B=2, T=10240, S=10240, Hq=16, Hkv=2, d=128, d_idx=64,
                        block=128, topk=8, dtype=bf, hot_blocks_per_group=3),
        # T < S, T % block = 40: pieces [0, 552), [552, 4648), [4648, 7208), [7208, 8232)
        "chunked_T_lt_S_offset": W("chunked_T_lt_S_offset", B=1, T=8232, S=8320, Hq=8, Hkv=2,
                                   d=128, d_idx=64, block=64, topk=6, dtype=bf),
        # one KV group; the 64-query piece [4608, 4672) merges into [4672, 5696)
        "chunked_merge_G1": W("chunked_merge_G1", B=1, T=5696, S=5696, Hq=8, Hkv=1, d=128,
                              d_idx=64, block=64, topk=6, dtype=bf),
        "whole_decode": W("whole_decode", B=4, T=1, S=8192, Hq=32, Hkv=8, d=128, d_idx=64,
                          block=64, topk=8, dtype=bf),
        "whole_fp32": _synth().WORKLOADS["tiny_fp32_prefill"],
        "whole_short_prefill": W("whole_short_prefill", B=2, T=1024, S=1024, Hq=8, Hkv=2,
                                 d=128, d_idx=64, block=128, topk=4, dtype=bf),
        "prefill_128k": _synth().WORKLOADS["prefill_128k"],
    }[name]


def _pinned_like(x):
    return torch.empty(x.shape, dtype=x.dtype, pin_memory=True)


def _run_both(w, seed=0):
    import block_sparse_long_03_b200 as msa
    inp = _synth().make_inputs(w, seed, device="cuda")
    dev = (inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V)
    O, lse, ids, ws = msa.forward(*dev, block=w.block, topk=w.topk)
    host_in = [x.cpu().pin_memory() for x in dev]
    hO, hlse, hids = _pinned_like(O), _pinned_like(lse), _pinned_like(ids)
    hO.fill_(7)
    hlse.fill_(7)
    hids.fill_(7)
    p = msa.params_from(inp.q_idx, inp.Q, inp.K, block=w.block, topk=w.topk)
    buf = msa.alloc_workspace(p, msa.MSA_WS_FORWARD_HOST)
    msa.msa_forward_host(p, *host_in, hids, hO, hlse, buf)
    torch.cuda.current_stream().synchronize()
    assert msa.msa_get_device_error(ws) == 0
    assert msa.msa_get_device_error(buf) == 0
    return inp, (O, lse, ids), (hO, hlse, hids)


@pytest.mark.parametrize("name", ["chunked_B2", "chunked_T_lt_S_offset", "chunked_merge_G1",
                                  "whole_decode", "whole_fp32", "whole_short_prefill",
                                  "prefill_128k"])
def test_host_call_equals_forward(name):
    w = _case(name)
    torch.cuda.empty_cache()
    inp, (O, lse, ids), (hO, hlse, hids) = _run_both(w)
    assert torch.equal(hids, ids.cpu()), f"{name}: ids differ"
    assert torch.equal(hlse.view(torch.int32), lse.cpu().view(torch.int32)), f"{name}: lse differs"
    assert torch.equal(hO.view(torch.int16) if w.dtype == torch.bfloat16 else hO,
                       (O.cpu().view(torch.int16) if w.dtype == torch.bfloat16 else O.cpu())), \
        f"{name}: O differs"
    if name == "chunked_B2":
        # sampled rows plus both sides of every chunk boundary
        edges = [b * w.T + t for b in range(w.B)
                 for t in (511, 512, 4607, 4608, 8703, 8704, 9215, 9216)]
        rows = sorted(set(_synth().sample_rows(w, 24)) | set(edges))
        ref = parity.oracle_rows(inp, w, rows)
        parity.assert_ids_equal(parity.gather_rows(hids, rows, w.T), ref["ids"], name)
        parity.assert_close(parity.gather_rows(hO, rows, w.T), parity.gather_rows(hlse, rows, w.T),
                            ref["O"], ref["lse"], w.dtype, name)
    del inp, O, lse, ids, hO, hlse, hids
    torch.cuda.empty_cache()


def test_host_call_rejects_pageable_buffers():
    import block_sparse_long_03_b200 as msa
    w = _case("whole_short_prefill")
    inp = _synth().make_inputs(w, 0, device="cpu")
    p = msa.params_from(inp.q_idx, inp.Q, inp.K, block=w.block, topk=w.topk)
    buf = msa.alloc_workspace(p, msa.MSA_WS_FORWARD_HOST)
    O = torch.empty_like(inp.Q)
    lse = torch.empty(inp.Q.shape[:3], dtype=torch.float32)
    with pytest.raises(msa.MsaError) as e:
        msa.msa_forward_host(p, inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, None, O, lse, buf)
    assert e.value.status == 1
