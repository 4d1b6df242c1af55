"""Multi-rank host logic of bench.py on CPU: two gloo ranks, each timing its
own replica of the workload. The job's device time is the slowest rank's,
and the job's throughput counts every rank's work (weak scaling)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [2.5, 3.25][rank]  # the ranks' own step times
        slowest = bench.max_over_ranks(ms, world, device="cpu")
        out[rank] = (slowest, bench.job_tflops(world, 1.0e12, slowest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_count_both_replicas():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    for r in range(world):
        slowest, tflops = res[r]
        assert slowest == 3.25
        # 2 ranks x 1e12 FLOP in 3.25 ms
        assert tflops == pytest.approx(2 * 1.0e12 / 3.25e-3 / 1e12)


def test_single_rank_is_the_identity():
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.job_tflops(1, 4.0e12, 2.0) == pytest.approx(2000.0)
