"""The five workloads at full size, in the launch configuration the benchmark
times (msa_forward on device-resident inputs), against the oracle on a
sample of rows; plus properties checked on EVERY row: each (row, group)
keeps exactly min(k, cb + 1) distinct ascending ids, all <= cb, with cb
among them, and LSE is finite."""
import numpy as np
import pytest
import torch

from tests import parity

pytestmark = pytest.mark.gpu

N_SAMPLE = {"tiny_fp32_prefill": 0, "prefill_32k": 48, "prefill_128k": 32, "decode_128k": 16,
            "chunked_prefill_1m": 32}


def _check_all_rows_valid(ids, w):
    B, T, G, k = ids.shape
    t = torch.arange(T, device=ids.device)
    cb = ((w.S - w.T + t) // w.block).view(1, T, 1)
    n_keep = torch.clamp(cb + 1, max=k)
    valid = ids >= 0
    assert torch.equal(valid.sum(-1), n_keep.expand(B, T, G)), "wrong number of kept ids"
    slot = torch.arange(k, device=ids.device).view(1, 1, 1, k)
    assert torch.equal(valid, (slot < n_keep.unsqueeze(-1)).expand_as(valid)), \
        "ids not packed at the front"
    big = torch.where(valid, ids, (1 << 30) + slot.expand_as(ids).to(ids.dtype))
    assert bool((big[..., 1:] > big[..., :-1]).all()), "ids not strictly ascending"
    assert bool((torch.where(valid, ids, cb.unsqueeze(-1)) <= cb.unsqueeze(-1)).all())
    last = ids.gather(-1, (n_keep - 1).unsqueeze(-1).expand(B, T, G, 1)).squeeze(-1)
    assert torch.equal(last, cb.expand(B, T, G)), "current block not kept"


@pytest.mark.parametrize("name", ["tiny_fp32_prefill", "prefill_32k", "prefill_128k",
                                  "decode_128k", "chunked_prefill_1m"])
def test_workload_full_size(name):
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import synthetic
    w = synthetic.WORKLOADS[name]
    torch.cuda.empty_cache()
    inp = synthetic.make_inputs(w, seed=0, device="cuda")
    O, lse, ids, ws = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                  topk=w.topk)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    _check_all_rows_valid(ids, w)
    assert bool(torch.isfinite(lse).all())
    n = N_SAMPLE[name]
    rows = list(range(w.B * w.T)) if n == 0 else synthetic.sample_rows(w, n)
    ref = parity.oracle_rows(inp, w, rows)
    parity.assert_ids_equal(parity.gather_rows(ids, rows, w.T), ref["ids"], name)
    parity.assert_close(parity.gather_rows(O, rows, w.T), parity.gather_rows(lse, rows, w.T),
                        ref["O"], ref["lse"], w.dtype, name)
    del inp, O, lse, ids, ws
    torch.cuda.empty_cache()
