"""The indexer's KL target (msa_forward_mass / msa_sparse_attn_fwd_mass:
each kept slot's share of the row's softmax, averaged over the group's
heads) against the fp64 oracle, on the tensor-core prefill path, the decode
path and the CUDA-core path; the extra output leaves O, LSE and ids
bitwise unchanged; masses sum to 1 per (row, group); skipped caller ids get
0; and the 128K prefill checked on every row (sums) and on sampled rows."""
import numpy as np
import pytest
import torch

from tests import parity
from tests.test_gpu_parity import _case, _dedup_valid, _inputs

pytestmark = pytest.mark.gpu

CASES = ["tiny_fp32_prefill", "fp32_gqa8", "bf16_prefill_2x1024", "bf16_chunk_ragged",
         "bf16_prefill_R16", "bf16_prefill_odd_blocks", "bf16_prefill_B2_chunk",
         "bf16_decode_small", "bf16_decode_T4", "bf16_decode_topk64", "bf16_decode_R16",
         "bf16_prefill_topk128", "bf16_decode_topk128", "bf16_d64_R8", "bf16_prefill_R16_topk64"]


def _msa():
    import block_sparse_long_03_b200 as msa
    return msa


def _check_mass(got, ids, ref_mass, dtype, where):
    tol = parity.MASS_TOL[dtype]
    d = np.abs(got.astype(np.float64) - ref_mass)
    assert d.max() <= tol, f"{where}: mass max err {d.max():.3g} (tol {tol:.3g})"
    assert np.all(got[ids < 0] == 0.0), f"{where}: an empty slot has mass"
    # 1 for every (row, group) that attends to a key, else 0
    sums, want = got.astype(np.float64).sum(-1), ref_mass.sum(-1)
    assert np.abs(sums - want).max() <= 1e-5, f"{where}: masses sum to {sums.min()}..{sums.max()}"
    return d.max()


@pytest.mark.parametrize("name", CASES)
def test_block_mass_matches_oracle(name):
    msa = _msa()
    w = _case(name)
    inp = _inputs(w, seed=1)
    O, lse, ids, mass, ws = msa.forward_with_mass(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V,
                                                  block=w.block, topk=w.topk)
    O2, lse2, ids2, ws2 = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V,
                                      block=w.block, topk=w.topk)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    assert torch.equal(ids, ids2)
    assert torch.equal(lse, lse2)
    assert torch.equal(O.float(), O2.float()), "the mass output changed O"
    rows = list(range(w.B * w.T)) if w.B * w.T <= 4096 else sorted(
        set(range(0, w.B * w.T, 13)) | {w.B * w.T - 1})
    ref = parity.oracle_rows(inp, w, rows)
    parity.assert_ids_equal(parity.gather_rows(ids, rows, w.T), ref["ids"], name)
    ref_mass = parity.oracle_mass_rows(inp, w, rows, ref["ids"], ref["lse"])
    _check_mass(parity.gather_rows(mass, rows, w.T), ref["ids"], ref_mass, w.dtype, name)


@pytest.mark.parametrize("name", ["bf16_chunk_ragged", "bf16_decode_small", "fp32_gqa8"])
def test_block_mass_with_bad_caller_ids(name):
    """Out-of-range and repeated caller ids are skipped: their slots get 0 and
    the other slots share the softmax of the valid blocks."""
    msa = _msa()
    w = _case(name)
    inp = _inputs(w, seed=5)
    O, lse, ids, ws = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                  topk=w.topk)
    bad = ids.clone()
    bad[..., -1] = w.NB + 7
    bad[..., 0] = bad[..., 1]
    p = msa.params_from(inp.q_idx, inp.Q, inp.K, block=w.block, topk=w.topk)
    O3, lse3 = torch.empty_like(O), torch.empty_like(lse)
    mass = torch.full(bad.shape, 7.0, dtype=torch.float32, device="cuda")
    wsa = msa.alloc_workspace(p, msa.MSA_WS_SPARSE_ATTN)
    msa.msa_sparse_attn_fwd_mass(p, inp.Q, inp.K, inp.V, bad, O3, lse3, mass, wsa)
    assert msa.msa_get_device_error(wsa) == 6
    valid = _dedup_valid(bad, w.NB)
    rows = list(range(0, w.B * w.T, 5))
    ref = parity.oracle_rows(inp, w, rows, ids=valid)
    ref_mass = parity.oracle_mass_rows(inp, w, rows, ref["ids"], ref["lse"])
    _check_mass(parity.gather_rows(mass, rows, w.T), ref["ids"], ref_mass, w.dtype, name)


def test_block_mass_prefill_128k():
    """The headline workload: masses sum to 1 on every (row, group), and
    match the oracle on sampled rows."""
    msa = _msa()
    from block_sparse_long_03_b200 import synthetic
    w = synthetic.WORKLOADS["prefill_128k"]
    torch.cuda.empty_cache()
    inp = synthetic.make_inputs(w, seed=0, device="cuda")
    O, lse, ids, mass, ws = msa.forward_with_mass(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V,
                                                  block=w.block, topk=w.topk)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    sums = mass.double().sum(-1)
    assert (sums - 1.0).abs().max().item() <= 1e-5
    assert bool((mass[ids < 0] == 0).all())
    rows = synthetic.sample_rows(w, 8)
    ref = parity.oracle_rows(inp, w, rows)
    parity.assert_ids_equal(parity.gather_rows(ids, rows, w.T), ref["ids"], "prefill_128k")
    ref_mass = parity.oracle_mass_rows(inp, w, rows, ref["ids"], ref["lse"])
    _check_mass(parity.gather_rows(mass, rows, w.T), ref["ids"], ref_mass, w.dtype,
                "prefill_128k")
    del inp, O, lse, ids, mass, ws
    torch.cuda.empty_cache()
