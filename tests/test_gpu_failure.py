"""Device failure path: a bounded wait that is never satisfied ends with an
error status the host reads, and the CUDA context stays usable (no trap, no
fault, no unbounded spin)."""
import time

import pytest
import torch

from tests import parity


@pytest.mark.gpu
def test_wait_timeout_reports_status_and_context_survives():
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import synthetic
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    msa.msa_selftest_wait_timeout(ws, 20000)            # 20 ms limit
    status = msa.msa_get_device_error(ws)
    elapsed = time.time() - t0
    assert status == 4, msa.status_string(status)        # MSA_ERR_DEVICE_TIMEOUT
    assert elapsed < 2.0
    assert msa.msa_get_device_error(ws) == 0             # reading clears the word
    # the context still runs the forward pass correctly
    w = synthetic.Workload("after_timeout", B=1, T=256, S=256, Hq=8, Hkv=2, d=128, d_idx=64,
                           block=64, topk=3, dtype=torch.bfloat16)
    inp = synthetic.make_inputs(w, 1, device="cpu")
    for f in ("q_idx", "k_idx", "Q", "K", "V"):
        setattr(inp, f, getattr(inp, f).cuda())
    O, lse, ids, ws2 = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                   topk=w.topk)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws2) == 0
    rows = list(range(w.T))
    ref = parity.oracle_rows(inp, w, rows)
    parity.assert_ids_equal(parity.gather_rows(ids, rows, w.T), ref["ids"], "after timeout")
    parity.assert_close(parity.gather_rows(O, rows, w.T), parity.gather_rows(lse, rows, w.T),
                        ref["O"], ref["lse"], w.dtype, "after timeout")


def test_selftest_rejects_bad_arguments_on_host():
    import ctypes
    from block_sparse_long_03_b200 import binding
    lib = binding.lib
    ws = ctypes.c_void_p(0x20000)                        # never touched
    assert lib.msa_selftest_wait_timeout(None, 256, 1000, None) == 5
    assert lib.msa_selftest_wait_timeout(ctypes.c_void_p(0x20010), 256, 1000, None) == 5
    assert lib.msa_selftest_wait_timeout(ws, 16, 1000, None) == 5
    assert lib.msa_selftest_wait_timeout(ws, 256, 0, None) == 1
    assert lib.msa_selftest_wait_timeout(ws, 256, 2000000, None) == 1
