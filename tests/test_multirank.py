"""The benchmark's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1 (one process per GPU in real runs).

Every rank runs its own batch of the same shape (the (sequence, value head) units shard without any exchange),
times it on its device, and the job's time is the slowest rank's; the whole-job throughput counts all ranks'
units.  These tests run that host logic with the gloo backend and CPU tensors.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from kda_gated_delta_prefill_b200 import inputs as gen


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's own time; every rank gets the maximum
        mine = 10.0 + 7.5 * rank
        got = bench.max_over_ranks(mine, world, "cpu")
        # each rank's own inputs for the same shape
        case = bench.rank_case(gen.SMALLEST, rank)
        x = gen.make_inputs(case)
        checksum = float(x["v"].float().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, (case.seed, checksum, tuple(x["q"].shape)))
        dist.barrier()
        out[rank] = (got, gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_inputs():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:  # no fork of this multi-threaded process
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in range(world):
        got, gathered = res[rank]
        assert got == pytest.approx(10.0 + 7.5 * (world - 1))  # the slowest rank's time, on every rank
        seeds = [gathered[r][0] for r in range(world)]
        assert len(set(seeds)) == world  # independent batches
        assert gathered[0][2] == gathered[1][2]  # of the same shape
        assert gathered[0][1] != gathered[1][1]


def test_single_rank_needs_no_group():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.rank_case(gen.SMALLEST, 0).seed == gen.SMALLEST.seed


def test_weak_scaling_throughput_counts_every_rank():
    # 4 ranks, each 1e6 token-heads per step, 10 steps in 20 ms on the slowest rank -> 2e9 token-heads/s
    assert bench.weak_throughput(1e6, 4, 20.0, 10) == pytest.approx(2e9)
    assert bench.weak_throughput(1e6, 1, 20.0, 10) == pytest.approx(5e8)
