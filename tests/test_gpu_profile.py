"""The per-kernel timing hook (msa_profile_begin/end) on the tensor-core
prefill path: one attention and one merge launch per row chunk are timed,
their sum stays within the call's own event time, and the outputs are
bitwise those of an unprofiled call."""
import pytest
import torch


@pytest.mark.gpu
def test_profile_counts_chunks_and_leaves_outputs_unchanged():
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import binding, synthetic
    w = synthetic.Workload("prof_16k", B=1, T=16384, S=16384, Hq=64, Hkv=8, d=128, d_idx=64,
                           block=128, topk=32, dtype=torch.bfloat16, hot_blocks_per_group=8)
    inp = synthetic.make_inputs(w, seed=1, device="cuda")
    ids = msa.topk_blocks(msa.index_block_scores(inp.q_idx, inp.k_idx, block=w.block), S=w.S,
                          block=w.block, topk=w.topk)
    O0, lse0, _ = msa.sparse_attn_fwd(inp.Q, inp.K, inp.V, ids, block=w.block)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    binding.msa_profile_begin()
    e0.record(s)
    O1, lse1, ws = msa.sparse_attn_fwd(inp.Q, inp.K, inp.V, ids, block=w.block)
    e1.record(s)
    torch.cuda.synchronize()
    r = binding.msa_profile_end()
    assert msa.msa_get_device_error(ws) == 0
    assert torch.equal(O0.view(torch.int16), O1.view(torch.int16))
    assert torch.equal(lse0, lse1)
    assert r["attn_launches"] >= 1 and r["attn_launches"] == r["merge_launches"]
    assert r["attn_ms"] > 0 and r["merge_ms"] > 0
    assert r["attn_ms"] + r["merge_ms"] <= e0.elapsed_time(e1) * 1.02
    # profiling is off again: a further call adds nothing
    binding.msa_profile_begin()
    r2 = binding.msa_profile_end()
    assert r2["attn_launches"] == 0
