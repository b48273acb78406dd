"""Host logic of the multi-GPU benchmark path, on CPU with two gloo ranks.

The decode path shards by sequence with no data-path collective; what runs
across ranks is the timing reduction (max over ranks) and the whole-job rate.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synthetic


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 3.0 * rank                     # the slowest rank sets the time
        ms_max = bench.max_over_ranks(ms, "cpu", world)
        rate = bench.whole_job_rate(1000.0, 5, world, ms_max)
        # per-rank inputs differ (seeded by rank) but share shapes
        inp = bench.bench_inputs(0, "cpu", rank)
        digest = float(inp["cache"].float().sum())
        q.put((rank, ms_max, rate, tuple(inp["cache"].shape), digest))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, v0, s0, d0), (r1, m1, v1, s1, d1) = res
    assert m0 == m1 == 13.0                        # max over ranks, on every rank
    assert v0 == v1 == pytest.approx(1000.0 * 5 * 2 / 0.013)
    assert s0 == s1
    assert d0 != d1


def _region_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per = 100.0 if rank == 0 else 40.0          # rank 1 needs 8 regions for 300 ms, rank 0 3
        calls = []

        def region():
            calls.append(1)
            dist.barrier()                          # as the timed region does: a mismatch would hang
            return per

        regions = bench.agreed_regions(region, 300.0, world, "cpu")
        dist.barrier()
        q.put((rank, len(regions), len(calls)))
    finally:
        dist.destroy_process_group()


def test_ranks_run_the_same_number_of_timed_regions():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_region_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 8, 8), (1, 8, 8)]


def test_single_rank_regions_stop_at_the_limit():
    per = iter([120.0, 120.0, 120.0, 120.0])
    assert bench.agreed_regions(lambda: next(per), 300.0, 1, "cpu") == [120.0, 120.0, 120.0]
    assert bench.agreed_regions(lambda: 500.0, 300.0, 1, "cpu") == [500.0]


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.5, "cpu", 1) == 7.5
    assert bench.whole_job_rate(131072, 10, 1, 2.0) == pytest.approx(131072 * 10 / 0.002)
