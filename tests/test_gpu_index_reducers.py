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
