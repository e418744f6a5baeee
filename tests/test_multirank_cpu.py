"""The multi-GPU path on the CPU: two gloo ranks take the slowest rank's time, as
bench.py does before it reports whole-job throughput (weak scaling, one replica of the
block per rank, no collective on the data path)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        t = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        out[rank] = t
    finally:
        dist.destroy_process_group()


def test_max_over_two_ranks():
    world, port = 2, _free_port()
    times = [1.25, 3.5]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, times, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1] == 3.5


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(2.0, 1, torch.device("cpu")) == 2.0
