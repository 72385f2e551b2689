"""The multi-GPU rule of the benchmark, on CPU with two gloo ranks.

The path does not shard: N GPUs run N independent replicas of the decode
step, and a multi-GPU number is the whole job's work over the slowest rank's
time.  These tests run the benchmark's own reduction (max over ranks) and
throughput formula in two processes joined by a gloo process group.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured these per-part times (ms); rank 1 is slower on part 0
        mine = [10.0 + 5.0 * rank, 3.0 - rank, 7.0]
        agg = bench.max_over_ranks(mine, dist)
        rate = bench.replica_rate(1000.0, agg[0] * 1e-3, world)
        out[rank] = (agg, rate)
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:   # no fork of a threaded process
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        results = dict(out)
    assert set(results) == {0, 1}
    for agg, rate in results.values():
        assert agg == [15.0, 3.0, 7.0]                 # element-wise max over the ranks
        assert rate == pytest.approx(1000.0 * 2 / 15e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.replica_rate(10.0, 2.0, 1) == 5.0
