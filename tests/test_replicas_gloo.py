"""The multi-GPU form of the forward is replicas: every rank runs its own
token batch with no collective on the data path, and the bench reports the
job's tokens over the slowest rank's time.  Its host logic (the max over
ranks, the whole-job throughput) runs here as world-size-2 gloo ranks on CPU.
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
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (1 + r) ms for its steps; every rank must see the slowest
        got = bench.reduce_max_over_ranks(1.0 + rank, torch.device("cpu"))
        # a second reduction in the same order on every rank
        got2 = bench.reduce_max_over_ranks(10.0 - rank, torch.device("cpu"))
        out[rank] = (got, got2)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert dict(out) == {0: (2.0, 10.0), 1: (2.0, 10.0)}


def test_max_over_ranks_without_group_is_identity():
    assert not dist.is_initialized()
    assert bench.reduce_max_over_ranks(3.25, torch.device("cpu")) == 3.25


@pytest.mark.parametrize("n,world,steps,ms", [(8192, 1, 300, 199.3), (8192, 2, 10, 2.0),
                                              (64, 8, 50, 3.35)])
def test_replica_throughput_counts_every_rank(n, world, steps, ms):
    """tokens of all ranks over the slowest rank's time: N ranks of the same
    time report N times one rank's throughput (weak scaling)."""
    v = bench.replica_tokens_per_s(n, world, steps, ms)
    assert v == pytest.approx(n * world * steps / (ms / 1000.0))
    assert v == pytest.approx(world * bench.replica_tokens_per_s(n, 1, steps, ms))
