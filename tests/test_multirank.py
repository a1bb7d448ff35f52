"""The multi-GPU path is independent replicas: each rank runs its own batch
and the job's throughput is every rank's tokens over the slowest rank's time.
Checked here on CPU with two gloo ranks (no GPU, no kernels)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = 100.0 + 50.0 * rank          # rank 1 is the slower replica
        ms, value = bench.job_throughput(ms_local, 32768 * 5, world, "cpu")
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_replica_throughput_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for ms, value in res.values():
        assert ms == 150.0                                  # the max over ranks
        assert value == pytest.approx(2 * 32768 * 5 / 0.150)


def test_single_rank_is_local():
    import bench
    ms, value = bench.job_throughput(200.0, 1000, 1, "cpu")
    assert ms == 200.0 and value == pytest.approx(5000.0)
