"""Host logic of bench.py's multi-GPU arm on CPU: two gloo ranks on
127.0.0.1 agree on the slowest rank's time, and the whole-job throughput of
N replicas counts every replica's work over that time."""
from __future__ import annotations

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "took" 1.5 + r ms; everyone must see the slowest
        out[rank] = bench.max_over_ranks(1.5 + rank, world, "cpu")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    import torch.multiprocessing as mp
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25


@pytest.mark.parametrize("world", [1, 2, 8])
def test_whole_job_throughput_counts_every_replica(world):
    sys.path.insert(0, ROOT)
    import bench
    flops, steps, ms = 1.9377e9, 500, 4.77
    one = bench.whole_job_tflops(1, flops, steps, ms)
    assert bench.whole_job_tflops(world, flops, steps, ms) == pytest.approx(world * one)
    assert one == pytest.approx(flops * steps / (ms * 1e-3) / 1e12)
