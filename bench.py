#!/usr/bin/env python
"""Benchmark of the MSA-style block-sparse attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one msa_forward over one batch of the 128K-token prefill
workload (B=1, T=S=131072, Hq=64, Hkv=8, d=128, d_idx=64, B_k=128, k=32,
bf16): index block scores, per-group Top-k with the current block kept,
sparse attention with LSE.  The 128K decode workload (64 sequences x 1
token, S=131072, Hq=32, Hkv=8, B_k=64, k=32) is timed the same way and
reported under "decode".  Inputs are synthetic, seeded, and resident in HBM
before timing; they are larger than L2 (126 MB), so no flush is needed.

With N > 1 (torchrun, one process per GPU) every rank runs its own
independent problem (weak scaling, no data-path collective); the time is the
max over ranks and `value` counts the tokens of all ranks.

`--impl reference` times the fp64 CPU oracle on the host cores on a bounded
row sample of the same workload (rank 0 only).

`roofline` names the dominant kernel, the tensor-core attention kernel: its
selected flops over its own launches, which the library brackets with CUDA
events on the call's stream during the timed steps (msa_profile_begin/end).
Beside it: the whole sparse-attention call (`call`), the merge kernels
(`merge`), the kernel's DRAM bytes per launch from a one-chunk ncu capture
(`traffic`, null once the attention source changes), and the time its
partial writes need at a write-only HBM rate measured in the same run
(`write_floor`).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL = "prefill_128k"
DECODE = "decode_128k"
METRIC = "MSA prefill tokens/s @128K"


# ---------------------------------------------------------------- accounting

def attended_keys(w) -> np.ndarray:
    """Causal keys each query attends under per-group Top-k with the current
    block kept: (kept blocks - 1) full blocks plus the causal part of the
    current block.  Shape [T]."""
    p = w.S - w.T + np.arange(w.T, dtype=np.int64)
    cb = p // w.block
    kept = np.minimum(w.topk, cb + 1)
    return (kept - 1) * w.block + (p - cb * w.block + 1)


def attention_flops(w) -> float:
    """4 d flops per (query head, attended key): QK^T and PV."""
    return float(w.B * w.Hq * 4 * w.d * attended_keys(w).sum())


def index_flops(w) -> float:
    """2 d_idx flops per (query, group, causal key)."""
    p = w.S - w.T + np.arange(w.T, dtype=np.int64)
    return float(w.B * w.G * 2 * w.d_idx * (p + 1).sum())


def kept_slots(w) -> int:
    """(query, group, kept slot) triples of a forward pass: min(k, cb + 1)
    per (query, group)."""
    p = w.S - w.T + np.arange(w.T, dtype=np.int64)
    return int(w.B * w.G * np.minimum(w.topk, p // w.block + 1).sum())


def partial_floor_bytes(w) -> float:
    """HBM bytes the KV-block-outer schedule of the sparse attention call must
    move whatever the kernels do: each (query, group, kept slot, head) partial
    (d bf16 values + an fp32 LSE) written once and read once by the combine,
    plus Q, K, V read once and O, LSE written once."""
    e = 2 if w.dtype == torch.bfloat16 else 4
    slots = kept_slots(w)
    partials = slots * (w.Hq // w.Hkv) * (w.d * 2 + 4) * 2
    io = w.B * w.T * w.Hq * (2 * w.d * e + 4) + 2 * w.B * w.S * w.G * w.d * e
    return float(partials + io)


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of the sparse
# attention call's main kernels, from a one-pass ncu capture of ONE row
# chunk (the fourth of five: rows 24195..32259, 8065 rows like every full
# chunk of the 128K call, every row keeping k blocks) of the workload
# `prefill_32k_h64` (the 128K prefill's heads, group size and k at 32K tokens;
# Q is larger than L2 as there):
#   python bench.py --workload prefill_32k_h64 --attn-call-once
# under ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,
# dram__bytes_write.sum -k regex:"attn_tc_kernel|merge_" -s 9 -c 3 (the
# attention kernel and the merge's two passes of that chunk).
# The figures are per kept (query, group) slot of the chunk; a call's traffic
# is that times its kept slots (the partials, the Q gather and the merge's
# reads all grow with the slots; K/V and the CSR kernels add < 1 %).  Held
# with the SHA-256 of the attention source: null once that source changes.
MEASURED_TRAFFIC = {
    "source": "block_sparse_long_03_b200/csrc/attn_tc.cu",
    "source_sha256": "48e6c5e6d6552623caadd10f200e69635c6a3ce5357985d69407dff41f7e161f",
    "workload": "prefill_32k_h64",
    "slots": 8065 * 8 * 32,                       # kept (row, group) slots of the chunk
    "kernels": {"attn_tc_kernel": {"read": 336722688.0, "write": 4236628480.0},
                "merge_weights_kernel": {"read": 74349056.0, "write": 6138368.0},
                "merge_apply_kernel": {"read": 4294501376.0, "write": 127399424.0}},
}


def measured_traffic(w):
    """(bytes, read, write) of one msa_sparse_attn_fwd call on workload `w`,
    scaled from the per-slot capture, or None."""
    import hashlib
    m = MEASURED_TRAFFIC
    if m is None:
        return None
    with open(os.path.join(ROOT, m["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != m["source_sha256"]:
            return None
    slots = kept_slots(w)
    rd = sum(k["read"] for k in m["kernels"].values()) / m["slots"] * slots
    wr = sum(k["write"] for k in m["kernels"].values()) / m["slots"] * slots
    per = {name: (k["read"] + k["write"]) / m["slots"] * slots for name, k in m["kernels"].items()}
    per_w = {name: k["write"] / m["slots"] * slots for name, k in m["kernels"].items()}
    return {"bytes": rd + wr, "read_bytes": rd, "write_bytes": wr, "from": m["workload"],
            "kernels": per, "kernel_writes": per_w}


def decode_bytes(w) -> float:
    """HBM bytes a decode step must move: all index keys, the kept K/V
    blocks, the index queries, Q, O, LSE, block scores and ids."""
    e = 2 if w.dtype == torch.bfloat16 else 4
    kept_tokens = attended_keys(w).sum()            # per (sequence, group)
    kv = w.B * w.G * kept_tokens * w.d * e * 2
    kidx = w.B * w.S * w.d_idx * e
    small = w.B * w.T * (w.G * w.d_idx * e + 2 * w.Hq * w.d * e + w.Hq * 4)
    bs = w.B * w.T * w.G * w.NB * 4 * 2 + w.B * w.T * w.G * w.topk * 4 * 2
    return float(kv + kidx + small + bs)


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons during a timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- GPU timing

def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=600),
            device_id=torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0"))))
    rank = int(os.environ.get("RANK", "0"))
    return rank, ws


def _barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def _max_over_ranks(x: float, ws: int) -> float:
    """The slowest rank's value (timing metadata only; no data-path exchange)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def workload_config(w, ws: int) -> dict:
    """The `config` of a bench line (the same in both arms)."""
    e = 2 if w.dtype == torch.bfloat16 else 4
    return {"workload": w.name, "B": w.B, "T": w.T, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv,
            "d": w.d, "d_idx": w.d_idx, "block": w.block, "topk": w.topk,
            "parallelism": f"replicas x{ws}",
            "l2": f"inputs larger than L2 (Q alone {w.B * w.T * w.Hq * w.d * e / 2**30:.1f} "
                  f"GiB); no flush"}


def rank_seed(rank: int) -> int:
    """Every rank works on its own independent problem (weak scaling)."""
    return 1000 * rank


def aggregate_tokens_per_s(tokens_per_rank: int, ms_max: float, ws: int) -> float:
    """Whole-job throughput: the tokens of all ranks over the slowest rank's time."""
    return ws * tokens_per_rank / (ms_max / 1e3)


class Problem:
    """Device-resident inputs, outputs and workspace of one workload."""

    def __init__(self, name: str, seed: int):
        import block_sparse_long_03_b200 as msa
        from block_sparse_long_03_b200 import synthetic
        self.msa = msa
        self.w = w = synthetic.WORKLOADS[name]
        self.inp = synthetic.make_inputs(w, seed, device="cuda")
        i = self.inp
        self.params = msa.params_from(i.q_idx, i.Q, i.K, block=w.block, topk=w.topk)
        self.O = torch.empty_like(i.Q)
        self.lse = torch.empty(i.Q.shape[:3], dtype=torch.float32, device="cuda")
        self.ids = torch.empty((w.B, w.T, w.G, w.topk), dtype=torch.int32, device="cuda")
        self.ws = None                  # msa_forward's workspace, on first use
        self.ws_attn = msa.alloc_workspace(self.params, msa.MSA_WS_SPARSE_ATTN)
        self.bs = None                  # the standalone calls' block scores, on first use
        self.mass = None

    def step(self, stream=None):
        i = self.inp
        if self.ws is None:
            self.ws = self.msa.alloc_workspace(self.params, self.msa.MSA_WS_FORWARD)
        self.msa.msa_forward(self.params, i.q_idx, i.k_idx, i.Q, i.K, i.V, self.ids, self.O,
                             self.lse, self.ws, stream)

    def step_mass(self, stream=None):
        """The forward pass plus the indexer's KL target (msa_forward_mass)."""
        i, w = self.inp, self.w
        if self.mass is None:
            self.mass = torch.empty((w.B, w.T, w.G, w.topk), dtype=torch.float32, device="cuda")
        if self.ws is None:
            self.ws = self.msa.alloc_workspace(self.params, self.msa.MSA_WS_FORWARD)
        self.msa.msa_forward_mass(self.params, i.q_idx, i.k_idx, i.Q, i.K, i.V, self.ids, self.O,
                                  self.lse, self.mass, self.ws, stream)

    def block_scores(self):
        w = self.w
        if self.bs is None:
            self.bs = torch.empty((w.B, w.T, w.G, w.NB), dtype=torch.float32, device="cuda")
        return self.bs

    def attn_call_once(self):
        """Index scores and Top-k as separate calls, then ONE msa_sparse_attn_fwd
        call (the launch sequence a profiler capture of that call selects from)."""
        m, i = self.msa, self.inp
        m.msa_index_block_scores(self.params, i.q_idx, i.k_idx, self.block_scores())
        m.msa_topk_blocks(self.params, self.bs, self.ids)
        torch.cuda.synchronize()
        m.msa_sparse_attn_fwd(self.params, i.Q, i.K, i.V, self.ids, self.O, self.lse,
                              self.ws_attn)
        torch.cuda.synchronize()
        return m.msa_get_device_error(self.ws_attn)

    def stage_times_ms(self, reps: int) -> dict:
        """Average device time of each call of the path, launched on its own."""
        m, i, s = self.msa, self.inp, torch.cuda.current_stream()
        self.block_scores()
        stages = {
            "index_block_scores": lambda: m.msa_index_block_scores(self.params, i.q_idx, i.k_idx,
                                                                   self.bs),
            "topk_blocks": lambda: m.msa_topk_blocks(self.params, self.bs, self.ids),
            "sparse_attn_fwd": lambda: m.msa_sparse_attn_fwd(self.params, i.Q, i.K, i.V, self.ids,
                                                             self.O, self.lse, self.ws_attn),
        }
        out = {}
        for name, fn in stages.items():
            fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(reps):
                fn()
            e1.record(s)
            torch.cuda.synchronize()
            out[name] = e0.elapsed_time(e1) / reps
        return out

    def free(self):
        for f in ("inp", "O", "lse", "ids", "ws", "ws_attn", "bs", "mass"):
            setattr(self, f, None)
        torch.cuda.empty_cache()


def index_reducers(prob, args, ws: int, kc: int) -> dict:
    """The index branch's cost at this shape, exact (msa_forward minus its
    attention call, which takes the same ids) against coarse-to-fine
    selection with kc candidates (msa_index_hierarchical), and the recall of
    the latter: the share of the exact selection's non-forced ids it keeps,
    over sampled rows."""
    m, i, w = prob.msa, prob.inp, prob.w
    steps = max(2, min(args.steps, 3))
    fwd_ms = time_steps(prob.step, steps, args.warmup, ws)
    attn_ms = time_steps(lambda: m.msa_sparse_attn_fwd(prob.params, i.Q, i.K, i.V, prob.ids,
                                                       prob.O, prob.lse, prob.ws_attn),
                         steps, args.warmup, ws)
    hids = torch.empty_like(prob.ids)
    hws = m.alloc_workspace(prob.params, m.MSA_WS_INDEX_HIER)
    hier_ms = time_steps(lambda: m.msa_index_hierarchical(prob.params, kc, i.q_idx, i.k_idx,
                                                          hids, hws),
                         steps, args.warmup, ws)
    prob.step()                                   # the exact ids of these inputs
    torch.cuda.synchronize()
    g = torch.Generator(device="cuda").manual_seed(3)
    rows = torch.randint(w.block * w.topk, w.T, (4096,), generator=g, device="cuda")
    ex = prob.ids[0, rows].long()                 # [n, G, k]; slot k - 1 is the current block
    hi = hids[0, rows].long()
    hit = (ex[..., :-1, None] == hi[..., None, :-1]).any(-1).float().mean().item()
    del hws
    return {"workload": w.name, "kc": kc, "exact_index_topk_ms": fwd_ms - attn_ms,
            "hierarchical_ms": hier_ms, "attention_ms": attn_ms, "forward_ms": fwd_ms,
            "speedup": (fwd_ms - attn_ms) / hier_ms,
            "recall_of_exact_ids": hit,
            "recall_rows": "4096 sampled rows with every slot filled (t >= block * k)"}


def paged_decode(prob, args, ws: int, page_size: int = 64) -> dict:
    """The same decode batch through msa_decode_paged: the cache is a pool of
    pages (the dense cache cut into page_size-token pages) reached through a
    random page table, with sequence lengths drawn uniformly from [S/2, S]
    (ragged, most not a multiple of the block).  Bytes per step count the
    index keys and kept K/V rows of each sequence's own length."""
    m, i, w = prob.msa, prob.inp, prob.w
    g = torch.Generator(device="cuda").manual_seed(11)
    n_pages = w.B * w.S // page_size
    table = torch.randperm(n_pages, generator=g, device="cuda").to(torch.int32).view(w.B, -1)
    lens = torch.randint(w.S // 2, w.S + 1, (w.B,), generator=g, device="cuda").to(torch.int32)
    kc = i.k_idx.view(n_pages, page_size, w.d_idx)
    Kc = i.K.view(n_pages, page_size, w.Hkv, w.d)
    Vc = i.V.view(n_pages, page_size, w.Hkv, w.d)
    pws = m.alloc_workspace(prob.params, m.MSA_WS_DECODE_PAGED)

    def step():
        m.msa_decode_paged(prob.params, lens, table, page_size, n_pages, i.q_idx, kc, i.Q, Kc, Vc,
                           prob.ids, prob.O, prob.lse, pws)

    us = time_steps(step, max(args.steps, 10), args.warmup, ws) * 1e3
    L = lens.long().cpu()
    e = 2
    kept_keys = 0
    for Lb in L.tolist():                            # per sequence: the forced block is partial
        cb = (Lb - 1) // w.block
        kept_keys += (min(w.topk, cb + 1) - 1) * w.block + (Lb - 1 - cb * w.block + 1)
    nbytes = (int(L.sum()) * w.d_idx * e + w.G * kept_keys * w.d * e * 2 +
              w.B * (w.G * w.d_idx * e + 2 * w.Hq * w.d * e + w.Hq * 4))
    del pws
    return {"page_size": page_size, "lengths": f"uniform in [{w.S // 2}, {w.S}]",
            "us_per_step": us, "bytes_per_step": float(nbytes),
            "frac": nbytes / (us / 1e6) / 1e9 / peaks()["hbm_gbs"]}


def time_steps(fn, steps: int, warmup: int, ws: int, around=None):
    """Device time per step (CUDA events on the launching stream, max over
    ranks).  `around` = (start, stop): called just before the first and just
    after the last timed step (e.g. the library's per-kernel timing hook)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(ws)
    torch.cuda.synchronize()
    if around:
        around[0]()
    e0.record(s)
    for _ in range(steps):
        fn()
    e1.record(s)
    torch.cuda.synchronize()
    if around:
        around[1]()
    _barrier(ws)
    return _max_over_ranks(e0.elapsed_time(e1) / steps, ws)


def e2e_prefill(prob: Problem, steps: int, warmup: int, ws: int) -> dict:
    """Same metric through the C-ABI call that takes HOST buffers
    (msa_forward_host): each step copies the inputs from pinned host memory,
    runs the forward pass and copies O and LSE back into pinned host memory,
    all inside the call (the copies overlap the kernels chunk by chunk)."""
    i = prob.inp
    m = prob.msa
    host_in = [x.cpu().pin_memory() for x in (i.q_idx, i.k_idx, i.Q, i.K, i.V)]
    host_O = torch.empty(prob.O.shape, dtype=prob.O.dtype, pin_memory=True)
    host_lse = torch.empty(prob.lse.shape, dtype=prob.lse.dtype, pin_memory=True)
    buf = m.alloc_workspace(prob.params, m.MSA_WS_FORWARD_HOST)

    def step():
        m.msa_forward_host(prob.params, *host_in, None, host_O, host_lse, buf)

    ms = time_steps(step, steps, warmup, ws)
    w = prob.w
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = host_O.numel() * host_O.element_size() + host_lse.numel() * host_lse.element_size()
    del buf
    # The same bytes copied with no kernels at all, both directions at once on
    # two streams: the floor the host link sets for this step.
    dev_in = (i.q_idx, i.k_idx, i.Q, i.K, i.V)
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def copies():
        cur = torch.cuda.current_stream()
        up.wait_stream(cur)
        down.wait_stream(cur)
        with torch.cuda.stream(up):
            for d_, h_ in zip(dev_in, host_in):
                d_.copy_(h_, non_blocking=True)
        with torch.cuda.stream(down):
            host_O.copy_(prob.O, non_blocking=True)
            host_lse.copy_(prob.lse, non_blocking=True)
        cur.wait_stream(up)
        cur.wait_stream(down)

    floor_ms = time_steps(copies, steps, warmup, ws)
    return {"value": aggregate_tokens_per_s(w.B * w.T, ms, ws), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": ms,
            "call": "msa_forward_host", "copy_only_ms": floor_ms,
            "frac_of_copy_floor": floor_ms / ms}


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(name: str, budget_s: float, max_rows: int = 4096, seed: int = 7,
                  host=None):
    """Run the fp64 oracle (as it stands) on seeded rows of the workload until
    about `budget_s` seconds of CPU work are done.  Returns (rows/s, rows,
    seconds, threads).  Inputs are generated on the host with the same recipe."""
    import oracle
    from block_sparse_long_03_b200 import synthetic
    w = synthetic.WORKLOADS[name]
    if host is None:
        host = synthetic.make_inputs(w, seed, device="cpu") if w.B * w.T * w.Hq * w.d < 3e9 \
            else None
    if host is None:
        raise RuntimeError("workload too large to generate on the host")
    rng = np.random.default_rng(seed)
    threads = oracle.num_threads()
    # every oracle call gets at least one row per thread (rows run in parallel)
    done, elapsed, batch = 0, 0.0, max(2, threads)
    while elapsed < budget_s and done < max_rows:
        rows = np.sort(rng.integers(0, w.B * w.T, size=batch))
        for b in np.unique(rows // w.T):
            ts = rows[rows // w.T == b] % w.T
            tt = torch.from_numpy(ts)
            t0 = time.perf_counter()
            oracle.forward(host.q_idx[b].index_select(0, tt), host.k_idx[b:b + 1],
                           host.Q[b].index_select(0, tt), host.K[b:b + 1], host.V[b:b + 1], ts,
                           T=w.T, block=w.block, topk=w.topk)
            elapsed += time.perf_counter() - t0
        done += batch
        batch = min(batch * 2, max(64, threads))
    return done / elapsed, done, elapsed, threads


def run_reference(args, rank: int, ws: int):
    if rank != 0:
        return
    from block_sparse_long_03_b200 import synthetic
    w = synthetic.WORKLOADS[args.workload]
    host = synthetic.make_inputs(w, 7, device="cpu")
    budget = float(os.environ.get("MSA_REF_STEP_SECONDS", "8"))
    for _ in range(args.warmup):
        oracle_sample(args.workload, 0.5, max_rows=1, host=host)
    rates, rows_total, secs_total, threads = [], 0, 0.0, 1
    for _ in range(args.steps):
        rate, rows, secs, threads = oracle_sample(args.workload, budget / max(args.steps, 1),
                                                  host=host)
        rates.append(rate)
        rows_total += rows
        secs_total += secs
    value = rows_total / secs_total
    sample = (f"{rows_total} seeded query rows of {w.name} (all {w.Hq} heads each), "
              f"{secs_total:.1f} s of oracle time")
    line = {
        "impl": "reference", "metric": METRIC if w.name == PREFILL else f"MSA tokens/s ({w.name})",
        "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs_total / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, ws),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


NOMINAL_BF16_TFLOPS, NOMINAL_HBM_GBS = 2250.0, 8000.0


def write_only_gbs(nbytes: int = 4 << 30, reps: int = 10) -> float:
    """HBM bandwidth of a plain write-only stream on this GPU (torch fill of a
    buffer larger than L2), measured with CUDA events: the reference for the
    attention kernel, whose DRAM traffic is almost all partial-output writes."""
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        buf.fill_(1)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        buf.fill_(1)
    e1.record(s)
    torch.cuda.synchronize()
    gbs = nbytes / (e0.elapsed_time(e1) / reps / 1e3) / 1e9
    del buf
    torch.cuda.empty_cache()
    return gbs


def roofline(w, pk, stages, prof, steps, attn_fl, idx_fl, fill_gbs=None) -> dict:
    """The dominant kernel's roofline.  At the prefill shapes that is the
    tensor-core attention kernel: its selected flops per launch over its own
    launch time, measured live in the timed steps; the whole sparse-attention
    call (CSR build, attention, merge) and the merge are reported beside it."""
    call_ms = stages["sparse_attn_fwd"]
    n_attn = prof.get("attn_launches", 0)
    if stages["index_block_scores"] > call_ms or n_attn == 0:
        # index-dominated shapes (or no tensor-core attention launch): whole calls
        dom = max(stages, key=stages.get)
        fl = idx_fl if dom == "index_block_scores" else attn_fl
        ach = fl / (stages[dom] / 1e3) / 1e12
        return {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"], "traffic": None,
                "traffic_note": "whole call timed: no per-kernel capture for this shape",
                "peak_source": pk["source"] + " bf16 burst (of " + pk["source"] + ")",
                "frac_of_nominal": ach / NOMINAL_BF16_TFLOPS, "stage_ms": stages}
    per_step = n_attn / steps                             # attention launches per step
    attn_ms = prof["attn_ms"] / steps                     # the kernel's time per step
    ach = attn_fl / (attn_ms / 1e3) / 1e12
    mt = measured_traffic(w)
    merge_ms = prof["merge_ms"] / steps
    merge_bytes = (sum(v for k, v in mt["kernels"].items() if k != "attn_tc_kernel") if mt else
                   partial_floor_bytes(w) / 2)            # read back once, O written once
    call_tf = attn_fl / (call_ms / 1e3) / 1e12
    return {
        "kernel": "attn_tc_kernel", "bound": "tensor", "achieved": ach,
        "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
        "traffic": None if mt is None else mt["kernels"]["attn_tc_kernel"] / per_step,
        "traffic_note": ("DRAM bytes per attention-kernel launch (average of the step's "
                         f"{per_step:.0f}), per kept slot from a one-chunk ncu capture on "
                         + (mt["from"] if mt else "-") + " times the step's kept slots"
                         if mt else "null: no capture of the current attention source"),
        "peak_source": pk["source"] + " bf16 burst (of " + pk["source"] + ")",
        "frac_of_nominal": ach / NOMINAL_BF16_TFLOPS,
        "kernel_ms_per_step": attn_ms, "launches_per_step": per_step,
        "timing": "CUDA events around each attention-kernel launch on the call's stream, "
                  "over the timed steps (msa_profile_begin/end)",
        "call": {"name": "msa_sparse_attn_fwd", "ms": call_ms, "tflops": call_tf,
                 "frac": call_tf / pk["bf16_tflops"],
                 "frac_of_nominal": call_tf / NOMINAL_BF16_TFLOPS,
                 "traffic": None if mt is None else float(mt["bytes"])},
        "merge": {"kernels": "merge_weights_kernel + merge_apply_kernel", "ms_per_step": merge_ms,
                  "bytes_per_step": float(merge_bytes),
                  "achieved_gbs": merge_bytes / (merge_ms / 1e3) / 1e9,
                  "frac_of_hbm": merge_bytes / (merge_ms / 1e3) / 1e9 / pk["hbm_gbs"]},
        # the kernel's DRAM traffic is almost all partial writes: their time at
        # the write-only bandwidth measured in the same run is a second floor
        "write_floor": None if (mt is None or not fill_gbs) else {
            "bytes_per_step": mt["kernel_writes"]["attn_tc_kernel"],
            "write_only_gbs": fill_gbs,
            "ms": mt["kernel_writes"]["attn_tc_kernel"] / (fill_gbs * 1e9) * 1e3,
            "frac": mt["kernel_writes"]["attn_tc_kernel"] / (fill_gbs * 1e9) * 1e3 / attn_ms},
        "stage_ms": stages,
        # the schedule's own floor: partials through HBM at the measured bandwidth
        "partial_traffic_floor": {
            "hbm_bytes": partial_floor_bytes(w),
            "ms_at_measured_hbm": partial_floor_bytes(w) / (pk["hbm_gbs"] * 1e9) * 1e3,
            "frac": (partial_floor_bytes(w) / (pk["hbm_gbs"] * 1e9) * 1e3) / call_ms},
        "index_tflops": idx_fl / (stages["index_block_scores"] / 1e3) / 1e12}


# ---------------------------------------------------------------- main

def run_ours(args, rank: int, ws: int):
    import block_sparse_long_03_b200 as msa
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    pk = peaks()
    prob = Problem(args.workload, seed=rank_seed(rank))
    w = prob.w
    launches0 = msa.msa_kernel_launches()
    prof = {}
    with ClockSampler(local) as clk:
        # the attention and merge kernels' own launches timed live over the
        # timed steps (events on the call's stream, summed by the library)
        ms = time_steps(prob.step, args.steps, args.warmup, ws,
                        around=(msa.msa_profile_begin, lambda: prof.update(msa.msa_profile_end())))
    timed_launches = msa.msa_kernel_launches() - launches0
    per_step = timed_launches / float(args.steps + args.warmup)
    value = aggregate_tokens_per_s(w.B * w.T, ms, ws)
    stages = prob.stage_times_ms(max(2, args.steps))
    attn_fl, idx_fl = attention_flops(w), index_flops(w)
    roof = roofline(w, pk, stages, prof, args.steps, attn_fl, idx_fl, write_only_gbs())
    # the indexer's KL target as a third output of the same pass
    kl_ms = time_steps(prob.step_mass, args.steps, args.warmup, ws)
    ref_ms = time_steps(prob.step, args.steps, args.warmup, ws)    # adjacent, same clocks
    kl = {"call": "msa_forward_mass", "ms_per_step": kl_ms, "extra_ms": kl_ms - ref_ms,
          "value": aggregate_tokens_per_s(w.B * w.T, kl_ms, ws), "unit": "tokens/s",
          "mass_bytes": int(prob.mass.numel() * 4)}
    e2e = None if args.no_e2e else e2e_prefill(prob, max(1, min(args.steps, 3)), 1, ws)
    prob.free()
    del prob

    decode = None
    if not args.no_decode:
        dp = Problem(args.decode_workload, seed=rank_seed(rank) + 1)
        with ClockSampler(local) as dclk:
            dms = time_steps(dp.step, max(args.steps, 10), args.warmup, ws)
        dst = dp.stage_times_ms(max(args.steps, 10))
        db = decode_bytes(dp.w)
        decode = {"workload": args.decode_workload, "us_per_step": dms * 1e3, "bytes_per_step": db,
                  "achieved_gbs": db / (dms / 1e3) / 1e9, "peak_gbs": pk["hbm_gbs"],
                  "frac": db / (dms / 1e3) / 1e9 / pk["hbm_gbs"],
                  "frac_of_nominal": db / (dms / 1e3) / 1e9 / NOMINAL_HBM_GBS, "stage_ms": dst,
                  "clocks": dclk.summary(), "paged": paged_decode(dp, args, ws)}
        dp.free()

    # the pages' own 1M-token shape (prefill, and decode steps of 16 sequences)
    long_ctx = None
    if not args.no_1m:
        long_ctx = {}
        p1 = Problem("prefill_1m", seed=rank_seed(rank) + 2)
        with ClockSampler(local) as c1:
            ms1 = time_steps(p1.step, max(2, min(args.steps, 3)), args.warmup, ws)
        long_ctx["prefill_1m"] = {
            "tokens_per_s": aggregate_tokens_per_s(p1.w.B * p1.w.T, ms1, ws),
            "ms_per_step": ms1, "attention_flops": attention_flops(p1.w),
            "index_flops": index_flops(p1.w), "clocks": c1.summary()}
        long_ctx["index_reducers"] = index_reducers(p1, args, ws, kc=64)
        p1.free()
        del p1
        d1 = Problem("decode_1m", seed=rank_seed(rank) + 3)
        with ClockSampler(local) as c2:
            dms1 = time_steps(d1.step, max(args.steps, 10), args.warmup, ws)
        db1 = decode_bytes(d1.w)
        long_ctx["decode_1m"] = {
            "us_per_step": dms1 * 1e3, "bytes_per_step": db1,
            "achieved_gbs": db1 / (dms1 / 1e3) / 1e9, "peak_gbs": pk["hbm_gbs"],
            "frac": db1 / (dms1 / 1e3) / 1e9 / pk["hbm_gbs"], "clocks": c2.summary()}
        d1.free()
        del d1

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rate, rows, secs, threads = oracle_sample(args.workload, args.cpu_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{rows} seeded query rows of {w.name}, {secs:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC if w.name == PREFILL else f"MSA tokens/s ({w.name})", "value": value,
            "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; Q/K/V ~ N(0,1), index q/k on a 1/4 grid, hot blocks)",
            "config": workload_config(w, ws),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "kl_target": kl,
            "gpu_launches": int(round(per_step * args.steps)),
            "clocks": clk.summary(), "decode": decode, "long_context": long_ctx,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=PREFILL)
    ap.add_argument("--decode-workload", default=DECODE)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-1m", action="store_true",
                    help="skip the 1M-token prefill and decode figures")
    ap.add_argument("--attn-call-once", action="store_true",
                    help="run one msa_sparse_attn_fwd call on --workload and exit "
                         "(the command a profiler capture of that call wraps)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        return
    if args.attn_call_once:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        prob = Problem(args.workload, seed=0)
        status = prob.attn_call_once()
        print(json.dumps({"attn_call_once": args.workload, "device_error": status}), flush=True)
        sys.exit(1 if status else 0)
    rank, ws = _dist()
    try:
        run_ours(args, rank, ws)
    finally:
        if ws > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
