"""msa_forward_noalloc: the forward pass for callers that cannot allocate
device memory (code running where cudaMalloc is unavailable or forbidden,
or a process whose device memory is owned by someone else).  Its scratch
is a fixed device array inside the library instead of a caller workspace.

Checked through the C ABI against msa_forward (the entry point that takes a
workspace), within the parity tolerance of the other GPU tests, on two
calls in a row with different inputs, so that contents left in the shared
scratch by the first call cannot leak into the second.  This file is
collected last so that a run stopping at the first failure has run every
other test already; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests import parity

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def test_noalloc_matches_forward_on_two_calls():
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import binding, synthetic
    lib = binding.lib
    w = synthetic.Workload("noalloc", B=2, T=384, S=512, Hq=16, Hkv=2, d=128, d_idx=64,
                           block=128, topk=3, dtype=torch.bfloat16, hot_blocks_per_group=1)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed in (11, 12):                      # two calls in a row
        inp = synthetic.make_inputs(w, seed, device="cuda")
        p = msa.params_from(inp.q_idx, inp.Q, inp.K, block=w.block, topk=w.topk)
        # reference: the workspace entry point
        O_ref, lse_ref, ids_ref, ws = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V,
                                                  block=w.block, topk=w.topk)
        # the no-allocation entry point, called through the C ABI
        O = torch.full_like(inp.Q, float("nan"))
        lse = torch.full(inp.Q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
        ids = torch.full((w.B, w.T, w.G, w.topk), -7, dtype=torch.int32, device="cuda")
        rc = lib.msa_forward_noalloc(ctypes.byref(p), _ptr(inp.q_idx), _ptr(inp.k_idx),
                                     _ptr(inp.Q), _ptr(inp.K), _ptr(inp.V), _ptr(ids), _ptr(O),
                                     _ptr(lse), stream)
        assert rc == 0, binding.status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(ids, ids_ref)
        rows = list(range(w.B * w.T))
        parity.assert_close(parity.gather_rows(O, rows, w.T), parity.gather_rows(lse, rows, w.T),
                            parity.gather_rows(O_ref, rows, w.T).astype(np.float64),
                            parity.gather_rows(lse_ref, rows, w.T).astype(np.float64),
                            w.dtype, f"noalloc seed {seed}")
        # ids kept only in the scratch (block_ids = NULL) give the same output
        O2 = torch.empty_like(inp.Q)
        lse2 = torch.empty_like(lse)
        rc = lib.msa_forward_noalloc(ctypes.byref(p), _ptr(inp.q_idx), _ptr(inp.k_idx),
                                     _ptr(inp.Q), _ptr(inp.K), _ptr(inp.V), None, _ptr(O2),
                                     _ptr(lse2), stream)
        assert rc == 0, binding.status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(O2, O) and torch.equal(lse2, lse)


def test_noalloc_many_groups():
    """32 GQA groups (more than the 16 the CUDA-core index tile took before it
    sized its query tile by the group count): ids bitwise those of
    msa_forward, O and lse within the bf16 tolerance."""
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import binding, synthetic
    lib = binding.lib
    w = synthetic.Workload("noalloc_g32", B=1, T=192, S=256, Hq=32, Hkv=32, d=128, d_idx=64,
                           block=64, topk=3, dtype=torch.bfloat16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    inp = synthetic.make_inputs(w, 21, device="cuda")
    p = msa.params_from(inp.q_idx, inp.Q, inp.K, block=w.block, topk=w.topk)
    O_ref, lse_ref, ids_ref, ws = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V,
                                              block=w.block, topk=w.topk)
    O = torch.empty_like(inp.Q)
    lse = torch.empty(inp.Q.shape[:3], dtype=torch.float32, device="cuda")
    ids = torch.empty((w.B, w.T, w.G, w.topk), dtype=torch.int32, device="cuda")
    rc = lib.msa_forward_noalloc(ctypes.byref(p), _ptr(inp.q_idx), _ptr(inp.k_idx), _ptr(inp.Q),
                                 _ptr(inp.K), _ptr(inp.V), _ptr(ids), _ptr(O), _ptr(lse), stream)
    assert rc == 0, binding.status_string(rc)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids_ref)
    rows = list(range(w.B * w.T))
    parity.assert_close(parity.gather_rows(O, rows, w.T), parity.gather_rows(lse, rows, w.T),
                        parity.gather_rows(O_ref, rows, w.T).astype(np.float64),
                        parity.gather_rows(lse_ref, rows, w.T).astype(np.float64),
                        w.dtype, "noalloc G=32")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import binding
    lib = binding.lib
    # block scores alone: 1 * 16384 * 8 * 128 * 4 B = 64 MiB > 32 MiB
    p = msa.make_params(B=1, T=16384, S=16384, Hq=32, Hkv=8, d=128, d_idx=64, block=128, topk=16,
                        dtype=torch.bfloat16)
    assert msa.msa_workspace_size(p, msa.MSA_WS_FORWARD) > (32 << 20)
    fake = ctypes.c_void_p(0x10000)            # never touched: the size check comes first
    rc = lib.msa_forward_noalloc(ctypes.byref(p), fake, fake, fake, fake, fake, None, fake, fake,
                                 None)
    assert rc == 5, binding.status_string(rc)
