"""The benchmark's accounting, on the CPU: the selected attention flops, the
index flops, the partial-traffic floor and the decode bytes, against brute
force counts on tiny shapes and against the workload figures worked out
independently for the scope table (attention 1.03e12 / 1.71e13 / 5.45e11,
index 5.50e11 / 8.80e12 / 2.19e12 flops for the 32K, 128K and chunked 1M
prefills; 1.61 GB a decode step); and the guard that drops the measured
traffic once the attention source changes."""
import importlib.util
import os

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _workloads():
    from block_sparse_long_03_b200 import synthetic
    return synthetic


def _brute_keys(w):
    """Attended keys of each query by enumeration: the current block plus the
    topk - 1 blocks before it (all of them when fewer), causal tokens only."""
    out = []
    for t in range(w.T):
        p = w.S - w.T + t
        cb = p // w.block
        kept = [cb] + list(range(max(0, cb - (w.topk - 1)), cb))
        out.append(sum(1 for n in kept for j in range(n * w.block, (n + 1) * w.block)
                       if j <= p))
    return np.array(out)


@pytest.mark.parametrize("shape", [dict(B=1, T=300, S=300, block=16, topk=4),
                                   dict(B=2, T=50, S=200, block=32, topk=3),
                                   dict(B=1, T=64, S=64, block=64, topk=8)])
def test_flops_and_floor_by_enumeration(bench, shape):
    W = _workloads().Workload
    w = W("t", Hq=8, Hkv=2, d=16, d_idx=8, dtype=torch.bfloat16, **shape)
    keys = _brute_keys(w)
    assert np.array_equal(bench.attended_keys(w), keys)
    assert bench.attention_flops(w) == w.B * w.Hq * 4 * w.d * keys.sum()
    causal = sum(w.S - w.T + t + 1 for t in range(w.T))
    assert bench.index_flops(w) == w.B * w.G * 2 * w.d_idx * causal
    slots = w.B * w.G * sum(min(w.topk, (w.S - w.T + t) // w.block + 1) for t in range(w.T))
    R = w.Hq // w.Hkv
    partials = slots * R * (2 * w.d + 4) * 2                 # written once, read once
    io = w.B * w.T * w.Hq * (2 * w.d * 2 + 4) + 2 * w.B * w.S * w.G * w.d * 2
    assert bench.partial_floor_bytes(w) == partials + io


@pytest.mark.parametrize("name,attn,idx", [("prefill_32k", 1.03e12, 5.50e11),
                                           ("prefill_128k", 1.71e13, 8.80e12),
                                           ("chunked_prefill_1m", 5.45e11, 2.19e12)])
def test_workload_flops(bench, name, attn, idx):
    w = _workloads().WORKLOADS[name]
    assert abs(bench.attention_flops(w) / attn - 1) < 0.01
    assert abs(bench.index_flops(w) / idx - 1) < 0.01


def test_decode_bytes(bench):
    w = _workloads().WORKLOADS["decode_128k"]
    b = bench.decode_bytes(w)
    assert abs(b / 1.61e9 - 1) < 0.01
    # the index keys and the kept K/V blocks are most of it
    kidx = w.B * w.S * w.d_idx * 2
    kv = w.B * w.G * w.topk * w.block * w.d * 2 * 2
    assert kidx + kv < b < (kidx + kv) * 1.01


def test_kept_slots(bench):
    W = _workloads().Workload
    w = W("t", B=2, T=50, S=200, Hq=8, Hkv=2, d=16, d_idx=8, block=32, topk=3,
          dtype=torch.bfloat16)
    want = w.B * w.G * sum(min(w.topk, (w.S - w.T + t) // w.block + 1) for t in range(w.T))
    assert bench.kept_slots(w) == want


def test_measured_traffic_guard(bench, monkeypatch):
    """The per-slot capture scales with a call's kept slots, and is dropped
    once the attention source no longer has the captured hash."""
    import hashlib
    src = "block_sparse_long_03_b200/csrc/attn_tc.cu"
    with open(os.path.join(ROOT, src), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    fake = {"source": src, "source_sha256": sha, "workload": "prefill_32k_h64", "slots": 1000,
            "kernels": {"attn_tc_kernel": {"read": 3000.0, "write": 5000.0},
                        "combine_kernel": {"read": 6000.0, "write": 500.0}}}
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", fake)
    w = _workloads().WORKLOADS["prefill_128k"]
    m = bench.measured_traffic(w)
    slots = bench.kept_slots(w)
    assert m is not None and abs(m["read_bytes"] - 9.0 * slots) < 1e-3 * slots
    assert abs(m["write_bytes"] - 5.5 * slots) < 1e-3 * slots
    assert m["bytes"] == m["read_bytes"] + m["write_bytes"]
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", dict(fake, source_sha256="0" * 64))
    assert bench.measured_traffic(w) is None



def test_roofline_uses_the_kernels_own_time(bench, monkeypatch):
    """The roofline names the attention kernel: selected flops over its own
    event-timed launches per step; traffic per launch from the per-slot
    capture; the whole call and the merge are reported beside it.  An
    index-dominated shape falls back to whole calls."""
    import hashlib
    src = "block_sparse_long_03_b200/csrc/attn_tc.cu"
    with open(os.path.join(ROOT, src), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    fake = {"source": src, "source_sha256": sha, "workload": "prefill_32k_h64", "slots": 1000,
            "kernels": {"attn_tc_kernel": {"read": 3000.0, "write": 5000.0},
                        "combine_kernel": {"read": 6000.0, "write": 500.0}}}
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", fake)
    w = _workloads().WORKLOADS["prefill_128k"]
    pk = {"bf16_tflops": 1600.0, "hbm_gbs": 6500.0, "source": "measured"}
    stages = {"index_block_scores": 6.0, "topk_blocks": 1.5, "sparse_attn_fwd": 40.0}
    prof = {"attn_ms": 5 * 22.0, "attn_launches": 5 * 17, "merge_ms": 5 * 15.0,
            "merge_launches": 5 * 17}
    fl = 1.7e13
    r = bench.roofline(w, pk, stages, prof, 5, fl, 8.8e12, fill_gbs=4000.0)
    assert r["kernel"] == "attn_tc_kernel" and r["launches_per_step"] == 17
    wf = r["write_floor"]
    assert abs(wf["bytes_per_step"] - 5.0 * bench.kept_slots(w)) < 1e-3 * bench.kept_slots(w)
    assert abs(wf["ms"] - wf["bytes_per_step"] / 4e12 * 1e3) < 1e-9 * wf["ms"]
    assert abs(wf["frac"] - wf["ms"] / 22.0) < 1e-12
    assert abs(r["achieved"] - fl / 22e-3 / 1e12) < 1e-6 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / 1600.0) < 1e-12
    assert abs(r["call"]["tflops"] - fl / 40e-3 / 1e12) < 1e-6 * r["call"]["tflops"]
    slots = bench.kept_slots(w)
    assert abs(r["traffic"] - 8.0 * slots / 17) < 1e-3 * slots
    assert abs(r["merge"]["bytes_per_step"] - 6.5 * slots) < 1e-3 * slots
    assert r["call"]["traffic"] == bench.measured_traffic(w)["bytes"]
    # index-dominated: whole calls, no per-kernel traffic
    r2 = bench.roofline(w, pk, dict(stages, index_block_scores=50.0), prof, 5, fl, 8.8e12)
    assert r2["kernel"] == "index_block_scores" and r2["traffic"] is None
    assert abs(r2["achieved"] - 8.8e12 / 50e-3 / 1e12) < 1e-6 * r2["achieved"]
