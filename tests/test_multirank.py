"""Multi-rank host logic of bench.py, run as two gloo ranks on the CPU.

With N GPUs the benchmark runs one replica of the workload per rank (the
(b, h) tiles are independent, so no data-path collective exists); the ranks
meet only to take the maximum of their timings.  These tests run that logic
with world_size 2 on the gloo backend: the max-over-ranks reduction, the
whole-job aggregate, distinct replica inputs per rank, and the reference arm
printing from rank 0 only.
"""
import contextlib
import io
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        # each rank reports different step times; every rank must see the maximum
        times = [1.0 + rank, 10.0 - 3 * rank, 0.5 * (rank + 1)]
        got = bench.max_over_ranks(times, world)

        # replica inputs: same shapes, different seeds per rank (forward and decode)
        w = workloads.WORKLOADS["tiny_loglinear"]
        q, _, _ = workloads.make_qkv(w, seed=bench.replica_seed(w, rank))
        wd = workloads.DECODE_WORKLOADS["decode_loglinear_4k"]
        qd, _, _, _, _, lens = workloads.make_decode_inputs(wd, seed=bench.replica_seed(wd, rank))
        sums = [0.0] * (2 * world)
        sums[rank] = float(q.float().sum())
        sums[world + rank] = float(qd.float().sum()) + float(lens.sum())
        t = torch.tensor(sums, dtype=torch.float64)
        dist.all_reduce(t)  # gather the checksums (sum of one-hot vectors)

        # the reference arm prints only on rank 0
        class _Args:
            steps = 1
            warmup = 0
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            if rank != 0:
                bench.run_reference(_Args(), w, rank, world)
        results[rank] = (got, [float(x) for x in t], out.getvalue())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings_and_keep_replicas_apart():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(results)
    expect = [max(1.0 + r for r in range(world)), max(10.0 - 3 * r for r in range(world)),
              max(0.5 * (r + 1) for r in range(world))]
    for r in range(world):
        got, sums, printed = res[r]
        assert got == pytest.approx(expect)
        assert sums[0] != sums[1]          # the two replicas hold different inputs
        assert sums[2] != sums[3]          # ... and different decode batches
        assert printed == ""               # rank 1 does not print a reference line


def test_single_rank_reduction_is_identity_and_aggregate_counts_every_rank():
    assert bench.max_over_ranks([3.0, 1.5], 1) == [3.0, 1.5]
    flops = 8.47e9
    one = bench.whole_job_tflops(flops, 1, 0.1)
    assert one == pytest.approx(flops / 1e-4 / 1e12)
    # weak scaling: N replicas in the same time do N times the work
    assert bench.whole_job_tflops(flops, 4, 0.1) == pytest.approx(4 * one)


def test_replica_seeds_are_distinct_and_rank0_keeps_the_workload_seed():
    w = workloads.WORKLOADS["loglinear_4k"]
    seeds = [bench.replica_seed(w, r) for r in range(8)]
    assert seeds[0] == w.seed
    assert len(set(seeds)) == 8
