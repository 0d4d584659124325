"""Seeded synthetic inputs for MSA-style block-sparse attention.

This module generates inputs only: it holds none of the method's arithmetic
(no scores, no selection, no softmax).  Tests, the benchmark and the smoke
check draw their inputs from here, and the same tensors feed both the CUDA
library and the fp64 oracle.

Value recipe (the pages fix no data, so these are stated choices):
  * Q, K, V ~ N(0, 1), drawn in the workload dtype;
  * index queries and keys q_idx, k_idx = randint[-4, 4] / 4, so that every
    index dot product is a multiple of 1/32 well inside fp32's exact range;
  * "hot" blocks (prefill workloads): a shared seeded direction u with
    entries +-1/sqrt(d_idx) (unit norm; +-1/8 for d_idx = 64, exact in bf16)
    is added to the index keys of every token of the hot blocks.  Each GQA
    group draws its own hot block ids without replacement; k_idx has no
    group axis, so the shift goes to the union of the groups' draws.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtype and value recipe."""
    name: str
    B: int
    T: int
    S: int
    Hq: int
    Hkv: int
    d: int
    d_idx: int
    block: int
    topk: int
    dtype: torch.dtype
    hot_blocks_per_group: int = 0

    @property
    def G(self) -> int:
        return self.Hkv

    @property
    def NB(self) -> int:
        return -(-self.S // self.block)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads.  Sizes follow the block-sparse attention benchmark
# settings: B_k = 128 and k blocks per query for prefill; a 64-sequence
# decode batch; a 1M-token chunked prefill.
WORKLOADS = {
    "tiny_fp32_prefill": Workload("tiny_fp32_prefill", B=1, T=2048, S=2048, Hq=8, Hkv=2, d=64,
                                  d_idx=32, block=64, topk=8, dtype=torch.float32),
    "prefill_32k": Workload("prefill_32k", B=1, T=32768, S=32768, Hq=32, Hkv=8, d=128,
                            d_idx=64, block=128, topk=16, dtype=torch.bfloat16,
                            hot_blocks_per_group=8),
    "prefill_128k": Workload("prefill_128k", B=1, T=131072, S=131072, Hq=64, Hkv=8, d=128,
                             d_idx=64, block=128, topk=32, dtype=torch.bfloat16,
                             hot_blocks_per_group=8),
    "decode_128k": Workload("decode_128k", B=64, T=1, S=131072, Hq=32, Hkv=8, d=128,
                            d_idx=64, block=64, topk=32, dtype=torch.bfloat16),
    "chunked_prefill_1m": Workload("chunked_prefill_1m", B=1, T=4096, S=1 << 20, Hq=32, Hkv=4,
                                   d=128, d_idx=64, block=128, topk=64, dtype=torch.bfloat16,
                                   hot_blocks_per_group=32),
    # The pages' own long-context shape (64 query heads, 4 KV heads, head
    # dimension 128, B_k = 128, k = 16) at 2^20 tokens: a full prefill, and
    # decode steps of 16 sequences (the decode batch is not stated; d_idx as
    # in the other workloads).
    "prefill_1m": Workload("prefill_1m", B=1, T=1 << 20, S=1 << 20, Hq=64, Hkv=4, d=128,
                           d_idx=64, block=128, topk=16, dtype=torch.bfloat16,
                           hot_blocks_per_group=8),
    "decode_1m": Workload("decode_1m", B=16, T=1, S=1 << 20, Hq=64, Hkv=4, d=128, d_idx=64,
                          block=128, topk=16, dtype=torch.bfloat16),
    # Reduced sizes of the same shapes, small enough for profiler captures
    # (a few GB on the device).
    "prefill_8k": Workload("prefill_8k", B=1, T=8192, S=8192, Hq=64, Hkv=8, d=128, d_idx=64,
                           block=128, topk=32, dtype=torch.bfloat16, hot_blocks_per_group=8),
    "decode_4x128k": Workload("decode_4x128k", B=4, T=1, S=131072, Hq=32, Hkv=8, d=128,
                              d_idx=64, block=64, topk=32, dtype=torch.bfloat16),
    "decode_16x128k": Workload("decode_16x128k", B=16, T=1, S=131072, Hq=32, Hkv=8, d=128,
                               d_idx=64, block=64, topk=32, dtype=torch.bfloat16),
    # The 128K prefill's heads, group size and k at 32K tokens: four row
    # chunks of the same size as the 128K call's, Q still larger than L2.
    "prefill_32k_h64": Workload("prefill_32k_h64", B=1, T=32768, S=32768, Hq=64, Hkv=8, d=128,
                                d_idx=64, block=128, topk=32, dtype=torch.bfloat16,
                                hot_blocks_per_group=8),
}


@dataclasses.dataclass
class Inputs:
    q_idx: torch.Tensor   # [B, T, G, d_idx]
    k_idx: torch.Tensor   # [B, S, d_idx]
    Q: torch.Tensor       # [B, T, Hq, d]
    K: torch.Tensor       # [B, S, Hkv, d]
    V: torch.Tensor       # [B, S, Hkv, d]
    hot_blocks: list      # per group: list of planted block ids
    hot_direction: torch.Tensor | None


def _grid(gen, shape, device):
    """randint[-4, 4] / 4 as float32 (exact)."""
    return torch.randint(-4, 5, shape, generator=gen, device=device).to(torch.float32).mul_(0.25)


def make_inputs(w: Workload, seed: int, device="cpu") -> Inputs:
    """Draw the inputs of workload `w` from seed `seed` on `device`.

    The result is a deterministic function of (w, seed, device type): the CPU
    and CUDA generators give different streams, so a (workload, seed) pair is
    always generated on the same kind of device when results are compared.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    B, T, S, G = w.B, w.T, w.S, w.G
    q_idx = _grid(gen, (B, T, G, w.d_idx), device)
    k_idx = _grid(gen, (B, S, w.d_idx), device)
    hot, u = [], None
    if w.hot_blocks_per_group > 0:
        sign = torch.randint(0, 2, (w.d_idx,), generator=gen, device=device)
        u = (sign.to(torch.float32) * 2 - 1) / math.sqrt(w.d_idx)
        mark = torch.zeros(w.NB, dtype=torch.bool, device=device)
        for _g in range(G):
            ids = torch.randperm(w.NB, generator=gen, device=device)[: w.hot_blocks_per_group]
            hot.append(sorted(ids.tolist()))
            mark[ids] = True
        tok = mark.repeat_interleave(w.block)[:S]
        k_idx[:, tok, :] += u
    dt = w.dtype
    Q = torch.randn((B, T, w.Hq, w.d), generator=gen, device=device, dtype=dt)
    K = torch.randn((B, S, w.Hkv, w.d), generator=gen, device=device, dtype=dt)
    V = torch.randn((B, S, w.Hkv, w.d), generator=gen, device=device, dtype=dt)
    return Inputs(q_idx.to(dt), k_idx.to(dt), Q, K, V, hot, u)


def sample_rows(w: Workload, n: int, seed: int = 1234) -> list:
    """Rows r = b * T + t for a sampled parity check: the first and last rows
    and rows at the first block boundary of the first and last batch entries,
    plus `n` seeded random rows."""
    g = torch.Generator().manual_seed(seed)
    rows = set()
    for b in sorted({0, w.B - 1}):
        base = b * w.T
        rows.update({base, base + w.T - 1})
        if w.T > 1:
            rows.add(base + min(w.T - 1, w.block - 1))
            rows.add(base + min(w.T - 1, w.block))
    total = w.B * w.T
    extra = torch.randint(0, total, (max(0, n),), generator=g).tolist()
    rows.update(extra)
    return sorted(rows)
