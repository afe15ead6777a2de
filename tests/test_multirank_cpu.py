"""The N>1 path of bench.py on CPU: two gloo ranks on 127.0.0.1.

The method shards by (b,h): the job is one problem whose heads are split into contiguous blocks,
one per rank; heads are independent (the K mean is per head), so there is no data-path
collective, and the job's time is the slowest rank's.  These tests exercise the host logic the
GPU run uses (the head split, max over ranks, whole-job throughput, per-rank inputs, the
reference arm's rank filter) without a GPU, and show with the oracle that the split reproduces
the single-rank result.
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


@pytest.mark.parametrize("bh,world", [(64, 2), (5, 2), (7, 3), (3, 4), (0, 2), (128, 8)])
def test_shard_heads_partitions_the_heads(bh, world):
    import bench
    blocks = [bench.shard_heads(bh, world, r) for r in range(world)]
    covered = [h for start, n in blocks for h in range(start, start + n)]
    assert covered == list(range(bh))  # contiguous, in rank order, every head once
    sizes = [n for _, n in blocks]
    assert max(sizes) - min(sizes) <= 1


def _rank_shard_main(rank: int, world: int, port: int, out):
    import numpy as np

    import bench
    import oracle
    import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # a global problem with an uneven head count; every rank draws it (it is small) and
        # runs the whole method on its own head block only
        w = W.Workload("shard_b1h5_n192_d64_causal", 1, 5, 192, 64, True, True, n_out=4, out_mag=20.0)
        q, k, v = W.make_qkv(w)
        start, n = bench.shard_heads(w.BH, world, rank)
        sl = slice(start, start + n)
        ref = oracle.sage_attn(q[:, sl], k[:, sl], v[:, sl], w.causal, w.sm_scale, per_block=True)
        shards = [None] * world
        dist.all_gather_object(shards, (start, ref["o16"].view(np.uint16)))
        if rank == 0:
            full = oracle.sage_attn(q, k, v, w.causal, w.sm_scale, per_block=True)["o16"].view(np.uint16)
            joined = np.concatenate([o for _, o in sorted(shards, key=lambda t: t[0])], axis=1)
            out["equal"] = bool(np.array_equal(joined, full))
            out["starts"] = [st for st, _ in shards]
    finally:
        dist.destroy_process_group()


def test_head_shards_reproduce_the_single_rank_output():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_shard_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    assert res["starts"] == [0, 3]
    assert res["equal"]
