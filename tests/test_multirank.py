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


# ---------------------------------------------------------------- data-parallel shards

def _oracle_shard_compute(h, W, vals, idx, T_total, chunk, tau):
    """Stands in, on CPU ranks, for the per-shard GPU computation: the oracle's
    loss and gradients of these rows as one shard of a batch of T_total."""
    import oracle
    loss, _, _ = oracle.forward(h.numpy(), W.numpy(), vals.numpy(), idx.numpy(), tau, T_norm=T_total)
    dH, dW = oracle.backward(h.numpy(), W.numpy(), vals.numpy(), idx.numpy(), tau, T_norm=T_total)
    return torch.tensor(loss, dtype=torch.float64), torch.from_numpy(dH), torch.from_numpy(dW)


def _dp_rank_main(rank, world, port, out, cases):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from chunked_kl_loss_chunk_b200 import dp, inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = []
        for T_total, d, V, K, tau, seed in cases:
            # every rank draws the same batch and keeps its own block of rows
            h, W, vals, idx = inputs.make_loss_inputs(T_total, d, V, K, dtype=torch.float64, seed=seed)
            sh = dp.shard_rows(T_total, world, rank)
            sl = slice(sh.row0, sh.row0 + sh.rows)
            loss, dH, dW = dp.shard_step(h[sl], W, vals[sl], idx[sl], T_total, 16, tau,
                                         compute=_oracle_shard_compute, dtype=torch.float64)
            res.append((sh, float(loss), dH.numpy(), dW.numpy()))
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_dp_shards_two_gloo_ranks_match_the_whole_batch():
    """Two CPU ranks, each with its block of a batch: after the all-reduce both
    hold the batch's loss and dW, and their dH rows tile the batch's dH, all as
    the oracle computes them on the whole batch at once.  Cases: an even split,
    an odd T_total (uneven blocks), and T_total = 1 (rank 1 holds no rows)."""
    import numpy as np
    import oracle
    from chunked_kl_loss_chunk_b200 import inputs
    cases = [(12, 8, 40, 4, 1.0, 3), (7, 8, 33, 3, 1.7, 4), (1, 8, 20, 2, 1.0, 5)]
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_dp_rank_main, args=(world, port, out, cases), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    for ci, (T_total, d, V, K, tau, seed) in enumerate(cases):
        h, W, vals, idx = inputs.make_loss_inputs(T_total, d, V, K, dtype=torch.float64, seed=seed)
        loss_o, _, _ = oracle.forward(h.numpy(), W.numpy(), vals.numpy(), idx.numpy(), tau)
        dH_o, dW_o = oracle.backward(h.numpy(), W.numpy(), vals.numpy(), idx.numpy(), tau)
        rows = 0
        for rank in range(world):
            sh, loss, dH, dW = res[rank][ci]
            assert sh.row0 == rows
            rows += sh.rows
            assert loss == pytest.approx(loss_o, rel=1e-12)
            np.testing.assert_allclose(dW, dW_o, rtol=1e-12, atol=1e-15)
            np.testing.assert_allclose(dH, dH_o[sh.row0:sh.row0 + sh.rows], rtol=1e-12, atol=1e-15)
        assert rows == T_total


def test_shard_rows_tile_the_batch():
    from chunked_kl_loss_chunk_b200 import dp
    for T_total in (0, 1, 5, 8, 33, 32768):
        for world in (1, 2, 3, 8):
            shards = [dp.shard_rows(T_total, world, r) for r in range(world)]
            assert shards[0].row0 == 0
            for a, b in zip(shards, shards[1:]):
                assert b.row0 == a.row0 + a.rows
            assert sum(s.rows for s in shards) == T_total
            assert max(s.rows for s in shards) - min(s.rows for s in shards) <= 1
    with pytest.raises(ValueError):
        dp.shard_rows(8, 2, 2)
