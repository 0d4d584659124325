"""Index-cost reducers (the LSA page, "LongCat Sparse Attention", Abstract,
items (2) cross-layer indexing and (3) hierarchical indexing), on the GPU
against the oracle.

Cross-layer reuse: the block ids one layer's index branch selected are
passed, unchanged, to msa_sparse_attn_fwd for the next layer's Q, K and V
(no index work for that layer); the output is the oracle's attention over
those same ids."""
import pytest
import torch

from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["bf16_prefill_2x1024", "bf16_decode_small", "tiny_fp32_prefill",
                                  "bf16_prefill_R16"])
def test_cross_layer_id_reuse(name):
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import synthetic
    from tests.test_gpu_parity import _case
    w = _case(name)
    layer1 = synthetic.make_inputs(w, 31, device="cpu")
    layer2 = synthetic.make_inputs(w, 32, device="cpu")
    for inp in (layer1, layer2):
        for f in ("q_idx", "k_idx", "Q", "K", "V"):
            setattr(inp, f, getattr(inp, f).cuda())
    O1, lse1, ids1, ws1 = msa.forward(layer1.q_idx, layer1.k_idx, layer1.Q, layer1.K, layer1.V,
                                      block=w.block, topk=w.topk)
    launches = msa.msa_kernel_launches()
    O2, lse2, ws2 = msa.sparse_attn_fwd(layer2.Q, layer2.K, layer2.V, ids1, block=w.block)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws2) == 0
    rows = list(range(w.B * w.T))
    ref = parity.oracle_rows(layer2, w, rows, ids=ids1)
    parity.assert_close(parity.gather_rows(O2, rows, w.T), parity.gather_rows(lse2, rows, w.T),
                        ref["O"], ref["lse"], w.dtype, f"{name} layer 2 on layer-1 ids")
    # layer 2 differs from what its own index branch would give
    O3, lse3, ids3, _ = msa.forward(layer2.q_idx, layer2.k_idx, layer2.Q, layer2.K, layer2.V,
                                    block=w.block, topk=w.topk)
    assert not torch.equal(ids3, ids1)
    assert msa.msa_kernel_launches() > launches


# Hierarchical (coarse-to-fine) selection: coarse score = index query . the
# block's mean index key, the kc - 1 best earlier blocks are rescored
# exactly, and the current block plus the topk - 1 best of them are kept.
# Bit-exact against the oracle's coarse-to-fine selection on every row.
HIER_CASES = [("bf16_prefill_2x1024", 6), ("bf16_chunk_ragged", 12),
              ("bf16_prefill_odd_blocks", 9), ("bf16_decode_topk64", 64),
              ("bf16_prefill_R1_didx128", 8), ("bf16_prefill_B2_chunk", 3)]


def _oracle_hier(inp, w, kc):
    import numpy as np
    import oracle as orc
    out = []
    for b in range(w.B):
        ts = np.arange(w.T, dtype=np.int64)
        out.append(orc.select_hierarchical(inp.q_idx[b].cpu(), inp.k_idx[b:b + 1].cpu(), ts,
                                           T=w.T, block=w.block, topk=w.topk, kc=kc))
    return np.concatenate(out)


@pytest.mark.parametrize("name,kc", HIER_CASES)
def test_hierarchical_selection_matches_oracle(name, kc):
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import synthetic
    from tests.test_gpu_parity import _case
    w = _case(name)
    inp = synthetic.make_inputs(w, 41, device="cpu")
    ids, ws = msa.index_hierarchical(inp.q_idx.cuda(), inp.k_idx.cuda(), block=w.block,
                                     topk=w.topk, kc=kc)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    ref = _oracle_hier(inp, w, kc)
    parity.assert_ids_equal(ids.cpu().numpy().reshape(-1, w.G, w.topk), ref, f"{name} kc={kc}")


def test_hierarchical_with_every_block_a_candidate_is_exact():
    """kc - 1 >= every row's cb: the selection is msa_forward's exactly."""
    import block_sparse_long_03_b200 as msa
    from block_sparse_long_03_b200 import synthetic
    from tests.test_gpu_parity import _case
    w = _case("bf16_prefill_2x1024")            # NB = 8
    inp = synthetic.make_inputs(w, 43, device="cuda")
    ids, ws = msa.index_hierarchical(inp.q_idx, inp.k_idx, block=w.block, topk=w.topk,
                                     kc=w.NB)
    O, lse, ids_exact, ws2 = msa.forward(inp.q_idx, inp.k_idx, inp.Q, inp.K, inp.V, block=w.block,
                                         topk=w.topk)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids_exact)


def test_hierarchical_at_1m_tokens():
    """The pages' 1M-token shape (64 query heads, 4 groups, k = 16) with 64
    candidates per (query, group): processed in query pieces; sampled rows
    bit-exact against the oracle, every row a valid selection."""
    import numpy as np
    import block_sparse_long_03_b200 as msa
    import oracle as orc
    from block_sparse_long_03_b200 import synthetic
    w = synthetic.WORKLOADS["prefill_1m"]
    g = torch.Generator(device="cuda").manual_seed(5)
    q_idx = (torch.randint(-4, 5, (1, w.T, w.G, w.d_idx), generator=g, device="cuda")
             .float().mul_(0.25).to(torch.bfloat16))
    k_idx = (torch.randint(-4, 5, (1, w.S, w.d_idx), generator=g, device="cuda")
             .float().mul_(0.25).to(torch.bfloat16))
    ids, ws = msa.index_hierarchical(q_idx, k_idx, block=w.block, topk=w.topk, kc=64)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    t = torch.arange(w.T, device="cuda")
    cb = (t // w.block).view(1, -1, 1)
    valid = ids >= 0
    assert torch.equal(valid.sum(-1), torch.clamp(cb + 1, max=w.topk).expand(1, w.T, w.G))
    assert torch.equal(ids.max(-1).values, cb.expand(1, w.T, w.G).to(ids.dtype))
    rows = synthetic.sample_rows(w, 4)
    ref = orc.select_hierarchical(q_idx[0, rows].cpu(), k_idx.cpu(), np.asarray(rows), T=w.T,
                                  block=w.block, topk=w.topk, kc=64)
    parity.assert_ids_equal(ids[0, rows].cpu().numpy(), ref, "prefill_1m hierarchical")
