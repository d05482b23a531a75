"""The multi-rank plumbing of bench.py on CPU: world size 2 over gloo.

Every rank runs its own denoise chunk (weak scaling, no data-path
collective); ranks only meet at the barrier and the max-over-ranks timing."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    dist.barrier()
    ms = bench.max_over_ranks(10.0 + rank, dist, torch.device("cpu"))
    value = bench.job_throughput(1e12, world, ms)
    out[rank] = (ms, value)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        ms, value = out[r]
        assert ms == 11.0  # the slowest rank's time
        assert value == pytest.approx(1e12 * world / 11e-3 / 1e12)


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    assert bench.job_throughput(2e12, 1, 1000.0) == pytest.approx(2.0)
