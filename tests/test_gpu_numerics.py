"""Numerical edge cases of the CUDA library against the fp64 oracle, on each
kernel family (tensor-core prefill, decode, CUDA-core fp32):

  * signed zeros: block scores of -0.0 are stored as +0.0 (scores compare
    as numbers, the oracle's sums start from +0.0), compared by bit pattern;
    Top-k treats -0.0 and +0.0 as a tie and keeps the lower block id;
  * a caller-chosen softmax scale;
  * V of large magnitude: scaling V by 2^20 (exact in bf16) scales O by
    exactly 2^20 and leaves the LSE bitwise unchanged (the partial outputs
    cannot overflow), and O / 2^20 still matches the oracle;
  * caller ids above the current block (no causal token) are skipped and
    counted in the device error word, with the result unchanged.

Tolerances as in tests/parity.py."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu

PATHS = {   # one case per attention / index kernel family
    "tensor_core": "bf16_prefill_2x1024",
    "decode": "bf16_decode_small",
    "decode_R16": "bf16_decode_R16",
    "cuda_core_fp32": "fp32_gqa8",
}


def _msa():
    import block_sparse_long_03_b200 as msa
    return msa


def _case(name):
    from tests.test_gpu_parity import _case as c
    return c(name)


def _inputs(w, seed=0):
    from block_sparse_long_03_b200 import synthetic
    inp = synthetic.make_inputs(w, seed, device="cpu")
    for f in ("q_idx", "k_idx", "Q", "K", "V"):
        setattr(inp, f, getattr(inp, f).cuda())
    return inp


def test_topk_signed_zero_ties():
    """Rows whose k-1 boundary falls among scores of -0.0 and +0.0: the kept
    ids are the oracle's (equal scores, lower id first), for the warp-per-row
    kernel and the CTA-per-row kernel (> 2048 blocks)."""
    msa = _msa()
    for (T, S, G, block, k) in [(300, 4096, 2, 64, 6), (4, 2048 * 128 + 1024, 1, 128, 9)]:
        NB = S // block
        g = torch.Generator().manual_seed(T)
        # a few positive scores, then a sea of signed zeros, then negatives
        base = torch.randint(-3, 4, (1, T, G, NB), generator=g).float()
        base[base > 1] = 0.0                      # many zeros
        sign = torch.randint(0, 2, base.shape, generator=g).bool()
        bs = torch.where((base == 0) & sign, torch.tensor(-0.0), base)
        assert bool((torch.signbit(bs) & (bs == 0)).any())
        ids = msa.topk_blocks(bs.cuda(), S=S, block=block, topk=k).cpu().numpy()
        rows = np.arange(T)
        ref = orc.select_blocks(bs[0].numpy().astype(np.float64), rows, T=T, S=S, block=block,
                                topk=k)
        parity.assert_ids_equal(ids[0], ref, f"signed zeros NB={NB}")


@pytest.mark.parametrize("path", ["tensor_core", "decode", "cuda_core_fp32"])
def test_index_negative_zero_scores(path):
    """Index queries of -0.0 against a block whose index keys are all
    positive: every product is -0.0, so a dot product summed in IEEE order is
    -0.0; the stored block score is +0.0, as the oracle's, bit for bit."""
    msa = _msa()
    w = _case(PATHS[path])
    inp = _inputs(w, seed=11)
    q, k = inp.q_idx.clone(), inp.k_idx.clone()
    q[:, ::3] = -0.0                              # every third query token
    k[:, : w.block] = 0.25                        # block 0: all positive keys
    bs = msa.index_block_scores(q, k, block=w.block)
    rows = list(range(w.B * w.T))
    inp.q_idx, inp.k_idx = q, k
    ref = parity.oracle_rows(inp, w, rows, want_scores=True)
    got = parity.gather_rows(bs, rows, w.T)
    zeroed = np.asarray(rows) % w.T % 3 == 0
    assert (ref["bs"][zeroed][:, :, 0] == 0).all()
    parity.assert_bits_equal(got, ref["bs"], path)
    ids = msa.topk_blocks(bs, S=w.S, block=w.block, topk=w.topk)
    parity.assert_ids_equal(parity.gather_rows(ids, rows, w.T), ref["ids"], path)


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("scale", [0.03125, 0.3])
def test_caller_softmax_scale(path, scale):
    msa = _msa()
    w = _case(PATHS[path])
    inp = _inputs(w, seed=4)
    O, lse, ids, ws = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                  topk=w.topk, scale=scale)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    rows = list(range(w.B * w.T))
    ref = parity.oracle_rows(inp, w, rows, scale=scale)
    parity.assert_ids_equal(parity.gather_rows(ids, rows, w.T), ref["ids"], path)
    parity.assert_close(parity.gather_rows(O, rows, w.T), parity.gather_rows(lse, rows, w.T),
                        ref["O"], ref["lse"], w.dtype, f"{path} scale={scale}")


@pytest.mark.parametrize("path", list(PATHS))
def test_large_magnitude_values(path):
    """|V| up to ~4e6: far past fp16's range, well inside bf16's."""
    msa = _msa()
    w = _case(PATHS[path])
    inp = _inputs(w, seed=6)
    big = 2.0 ** 20
    O, lse, ids, ws = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                  topk=w.topk)
    V2 = inp.V * big                               # exact: a power of two
    assert float(V2.abs().max()) > 65504 * 16
    O2, lse2, ids2, ws2 = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, V2, block=w.block,
                                      topk=w.topk)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws2) == 0
    assert bool(torch.isfinite(O2.float()).all())
    assert torch.equal(ids2, ids)
    assert torch.equal(lse2, lse)
    assert torch.equal(O2, O * big), "O does not scale exactly with V"
    rows = list(range(0, w.B * w.T, 3))
    ref = parity.oracle_rows(inp, w, rows)
    parity.assert_close(parity.gather_rows(O2, rows, w.T) / big,
                        parity.gather_rows(lse2, rows, w.T), ref["O"], ref["lse"], w.dtype,
                        f"{path} V*2^20")


@pytest.mark.parametrize("name", ["bf16_prefill_2x1024", "tiny_fp32_prefill"])
def test_non_causal_caller_ids_counted(name):
    """An id above the row's current block (in range, no causal token) in an
    empty slot: skipped, recorded as MSA_ERR_BAD_BLOCK_IDS, and O / lse are
    bitwise those of the ids without it."""
    msa = _msa()
    w = _case(name)
    inp = _inputs(w, seed=8)
    O, lse, ids, ws = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                  topk=w.topk)
    torch.cuda.synchronize()
    t = torch.arange(w.T, device="cuda")
    cb = (w.S - w.T + t) // w.block
    planted = ids.clone()
    rows_with_room = (cb + 1 < w.topk) & (cb + 1 < w.NB)
    assert bool(rows_with_room.any())
    last = planted[..., -1]
    planted[..., -1] = torch.where(rows_with_room.view(1, -1, 1), (cb + 1).view(1, -1, 1).to(
        torch.int32).expand_as(last), last)
    assert not torch.equal(planted, ids)
    O2, lse2, ws2 = msa.sparse_attn_fwd(inp.Q, inp.K, inp.V, planted, block=w.block)
    O3, lse3, ws3 = msa.sparse_attn_fwd(inp.Q, inp.K, inp.V, ids, block=w.block)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws2) == 6
    assert msa.msa_get_device_error(ws3) == 0
    assert torch.equal(lse2, lse3) and torch.equal(O2, O3)


@pytest.mark.parametrize("NB,k,ties", [(4100, 17, False), (4099, 100, False), (2052, 33, True),
                                       (8192, 65, False), (3000, 66, True)])
def test_topk_long_rows(NB, k, ties):
    """Rows of more than 2048 blocks (the streaming warp kernel): threshold
    path (k - 1 <= 64), radix path (k - 1 > 64 or heavy ties), 16-byte and
    scalar row loads (NB % 4), against the oracle's selection."""
    msa = _msa()
    block, T, G = 64, 6, 2
    S = NB * block
    g = torch.Generator().manual_seed(NB + k)
    if ties:
        bs = (torch.randint(-2, 3, (1, T, G, NB), generator=g) * 0.5).float()
    else:
        bs = torch.randn((1, T, G, NB), generator=g).float()
    ids = msa.topk_blocks(bs.cuda(), S=S, block=block, topk=k).cpu().numpy()
    rows = np.arange(T)
    ref = orc.select_blocks(bs[0].numpy().astype(np.float64), rows, T=T, S=S, block=block, topk=k)
    parity.assert_ids_equal(ids[0], ref, f"long rows NB={NB} k={k}")
