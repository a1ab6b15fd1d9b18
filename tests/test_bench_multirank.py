"""The benchmark's multi-rank host logic on CPU with two gloo ranks: the
timing is the slowest rank's (every rank gets it), the whole-job rate counts
every rank's problem, ranks draw independent inputs, and the reference arm
runs on rank 0 only."""

import argparse
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_sparse_linear_mean_b200 import synth  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # the slowest rank's time, on every rank
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        assert ms == 10.0 + 5.0 * (world - 1), ms
        # whole-job rate: world problems of 1e12 flops x 4 steps in 20 ms
        assert abs(bench.job_rate(world, 1e12, 4, 20.0) - world * 200.0) < 1e-9
        # independent problems: rank r draws its inputs with seed r
        wl = synth.small_case(d=64, grid=(1, 2, 64))
        x = synth.make_inputs(wl, seed=rank, device="cpu")
        s = x.q.double().sum().reshape(1)
        allv = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allv, s)
        assert len({float(v) for v in allv}) == world
        # the reference arm: rank 0 alone runs; the others return at once
        if rank != 0:
            args = argparse.Namespace(workload="tiny", steps=1, warmup=3, gpus=world)
            assert bench.run_reference(args, rank, world) is None
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mp.spawn(rank_main, args=(world, free_port()), nprocs=world, join=True)


def test_single_process_reduction_is_the_value_itself():
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
