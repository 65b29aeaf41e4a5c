"""The bench's aggregation over ranks, on 2 gloo processes on the CPU: every rank gets the
slowest rank's time, and the whole-job throughput counts every rank's work over that time."""

import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = [0.5, 0.8, 0.6][rank]
        slowest = bench.max_over_ranks(ms, world, torch.device("cpu"))
        value = bench.whole_job_tflops(world, 5.498e11, slowest)
        np.save(os.path.join(out_dir, f"r{rank}.npy"), np.array([slowest, value]))
    finally:
        dist.destroy_process_group()


def test_slowest_rank_and_whole_job_value(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        slowest, value = np.load(tmp_path / f"r{r}.npy")
        assert slowest == 0.8
        assert abs(value - 2 * 5.498e11 / 0.8e-3 / 1e12) < 1e-9


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.7, 1, "cpu") == 0.7
    assert abs(bench.whole_job_tflops(1, 5.498e11, 0.55) - 999.6363636) < 1e-6


def test_workload_helpers():
    """The FLOP count the lines divide by, and the packed workload's lengths."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.attn_flops(2, 16, 8192, 128, True) == 5.497558138880e11  # 4 B H N^2 d / 2
    assert bench.attn_flops(1, 1, 4, 2, False) == 4 * 16 * 2
    w = bench.VARLEN_WORKLOAD
    lens = bench.varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
    assert sum(lens) == w["total"] and all(0 < n <= w["hi"] for n in lens)
    assert lens == bench.varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])  # seeded
