"""The multi-process (N > 1) path of the benchmark, on CPU with gloo: every
rank runs its own independent problem and only timing metadata is reduced
(the max over ranks); the whole-job value counts all ranks' tokens."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        local_ms = 10.0 * (rank + 1)                    # rank 1 is the slowest
        bench._barrier(world)
        ms = bench._max_over_ranks(local_ms, world)
        value = bench.aggregate_tokens_per_s(131072, ms, world)
        out[rank] = (ms, value, bench.rank_seed(rank))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_aggregate():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 20.0               # both ranks see the slowest time
    assert out[0][1] == out[1][1] == pytest.approx(2 * 131072 / 0.020)
    assert out[0][2] != out[1][2]                       # independent problems


def test_single_rank_is_identity():
    bench = _bench()
    assert bench._max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_tokens_per_s(1000, 1.0, 1) == pytest.approx(1e6)
