"""The N > 1 host path of bench.py on CPU: two gloo ranks.

More than one GPU runs independent replicas (each rank its own sequences, no
data-path collective); the job time is the slowest rank's and the job's
throughput counts every rank's tokens.  This checks that host logic with the
gloo backend -- the same calls bench.py makes over NCCL.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from long_context_decode_dual_b200 import workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 40.0][rank]
        m = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        wl = bench.rank_workload(W.workload("llama8b_b8_32k", n_ctx=64, batch=1), rank)
        K, _ = W.make_kv(wl)
        out.put((rank, m, bench.job_throughput(1000.0, m, world), wl.seed, float(np.asarray(K, np.float64).sum())))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_distinct_sequences():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, v0, s0, k0), (r1, m1, v1, s1, k1) = res
    assert m0 == m1 == 40.0                      # max over ranks
    assert v0 == v1 == pytest.approx(2 * 1000.0 / 0.040)
    assert s0 != s1 and k0 != k1                 # replicas decode different sequences


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    wl = W.workload("longctx_b1_128k")
    assert bench.rank_workload(wl, 0) is wl
