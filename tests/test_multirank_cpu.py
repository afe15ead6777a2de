"""The N>1 path of bench.py on CPU: two gloo ranks on 127.0.0.1.

The method shards by (b,h): every rank runs its own independent batch, there is no data-path
collective, and the job's time is the slowest rank's.  These tests exercise the host logic the
GPU run uses (max over ranks, whole-job throughput, per-rank inputs, the reference arm's rank
filter) without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import bench
    import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms_local, world, torch.device("cpu"))
        value = bench.job_tops(world, 1e12, ms_max)
        # per-rank inputs: seed = rank, so the ranks' batches differ
        q, _, _ = W.make_qkv(W.TINY, seed=rank)
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, q.double().sum().reshape(1))
        out[rank] = (ms_max, value, [float(x) for x in sums])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    for rank in range(world):
        ms_max, value, sums = res[rank]
        assert ms_max == 15.0                                   # the slow rank decides
        assert value == pytest.approx(world * 1e12 / 15e-3 / 1e12)  # both ranks' work over that time
        assert sums[0] != sums[1]                               # independent batches


def test_single_rank_helpers_need_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.job_tops(1, 2e12, 1000.0) == pytest.approx(2.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import argparse

    import bench
    import workloads as W
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(steps=1, warmup=3)
    assert bench.run_reference(args, W.TINY) is None  # other ranks exit without work
