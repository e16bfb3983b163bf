"""The multi-rank host path of bench.py on CPU (gloo, world size 2).

Tokens are independent, so the forward shards with no data-path collective:
every rank runs the full workload on its own GPU (weak scaling) and the job is
timed by its slowest rank.  These tests check that reduction and the aggregate
throughput with real gloo ranks, without a GPU.
"""
from __future__ import annotations

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


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench = _bench()
        assert bench.dist_info() == (world, rank, rank)
        elapsed = 10.0 + 5.0 * rank                 # rank 1 is the slowest
        mx = bench.reduce_max(elapsed, torch.device("cpu"))
        value = bench.aggregate_tokens_per_s(world, 4, 1000, mx)
        dist.barrier()
        q.put((rank, mx, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, mx, value in got:
        assert mx == 15.0
        assert value == pytest.approx(2 * 4 * 1000 / 0.015)


def test_single_process_reduction_is_identity():
    bench = _bench()
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    assert bench.aggregate_tokens_per_s(1, 10, 200704, 700.0) == pytest.approx(10 * 200704 / 0.7)
