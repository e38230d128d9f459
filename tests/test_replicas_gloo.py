"""The multi-GPU path is replicas only: every rank runs the same problem and the
benchmark reports the work of all ranks over the slowest rank's time.  Its
host-side aggregation runs here as two gloo ranks on the CPU."""
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


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = [2.0, 3.5][rank]                      # rank 1 is the slow one
        rate, ms = bench.replica_throughput(137.47, ms_local, True, torch.device("cpu"))
        out[rank] = (rate, ms)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replica_throughput_uses_slowest_rank_and_all_work():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    for rank in range(world):
        rate, ms = out[rank]
        assert ms == pytest.approx(3.5)
        assert rate == pytest.approx(world * 137.47 / 3.5e-3)


def test_single_process_needs_no_process_group():
    import bench
    rate, ms = bench.replica_throughput(10.0, 4.0, False, torch.device("cpu"))
    assert ms == 4.0 and rate == pytest.approx(2500.0)
