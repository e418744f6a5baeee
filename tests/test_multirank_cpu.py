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


def test_reference_arm_under_torchrun_prints_one_line():
    """bench.py --impl reference launched the way the driver launches N > 1 (torchrun, two
    ranks): rank 0 alone times the oracle and prints one JSON line, every rank exits 0."""
    import json
    import os
    import socket
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0", "--workload", "decode"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2
