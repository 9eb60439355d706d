"""The multi-rank bookkeeping of bench.py on CPU (two gloo ranks): every rank runs its
own replica, the job time is the max over ranks, and the throughput is the weak-scaling
sum. The path needs no data-path collective, so this is all that runs across ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
    job_ms = bench.max_over_ranks(ms, dist, "cpu")
    tops = bench.weak_scaling_tops(8.8e12, 3, world, job_ms)
    out[rank] = (job_ms, tops)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        job_ms, tops = out[r]
        assert job_ms == pytest.approx(15.0)
        assert tops == pytest.approx(2 * 8.8e12 * 3 / 15e-3 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.5) == 7.5
    assert bench.weak_scaling_tops(1e12, 2, 1, 1000.0) == pytest.approx(2.0)


def test_end_to_end_bound_from_the_input_copy():
    """The e2e ceiling: the step's input bytes over the measured copy time."""
    b = bench._e2e_bound(8.8e12, 1, 805306368, 14.5)
    assert b["h2d_gbs"] == pytest.approx(805306368 / 14.5e-3 / 1e9)
    assert b["h2d_bound"] == pytest.approx(8.8e12 / 14.5e-3 / 1e12)
    assert bench._e2e_bound(8.8e12, 4, 805306368, 14.5)["h2d_bound"] == pytest.approx(
        4 * 8.8e12 / 14.5e-3 / 1e12)
