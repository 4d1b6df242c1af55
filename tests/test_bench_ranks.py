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


def test_reference_arm_prints_the_contract_line_with_the_gpu_arms_config():
    """The reference arm (the oracle on the host cores) on a small workload:
    one JSON line with impl=reference, the same config dict the GPU arm
    prints, the cpu_baseline description of this run and an e2e entry with no
    host-device traffic."""
    import json
    import subprocess
    import sys

    from bit_attention_diffusion_b200 import synth
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny_b1h2n1024"],
                       capture_output=True, text=True, timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    wl, _ = synth.make_by_name("tiny_b1h2n1024")
    assert line["impl"] == "reference"
    assert line["config"] == bench.bench_config(wl, "e4m3", 1)
    assert line["unit"] == "TFLOPS" and line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and "head" in line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
