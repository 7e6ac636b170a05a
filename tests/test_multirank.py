"""The multi-GPU plumbing of bench.py (one process per GPU, weak scaling,
timing taken as the max over ranks) exercised with two gloo ranks on CPU."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w, r, local = bench.dist_setup(world, backend="gloo")
    try:
        assert (w, r, local) == (world, rank, rank)
        bench.barrier(w)
        # each rank reports a different time; everyone must see the slowest
        t = bench.max_over_ranks(10.0 + 5.0 * rank, w)
        out[rank] = (t, bench.rank_seed(r))
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_batches():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0          # max over ranks
    assert out[0][1] != out[1][1]                  # each rank its own batch


def test_job_throughput_counts_all_ranks():
    f = bench.flops(4, 16, 8192, 128, False)
    assert bench.job_throughput(f, 1, 2.0) * 2 == pytest.approx(bench.job_throughput(f, 2, 2.0))
    assert bench.job_throughput(f, 1, 2.0) == pytest.approx(f / 2e-3 / 1e12)
    assert bench.flops(1, 1, 128, 64, True) * 2 == bench.flops(1, 1, 128, 64, False)
