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


class _DoneProcess:
    def terminate(self):
        pass

    def wait(self):
        return 0


def test_clock_record_median_and_reasons(tmp_path):
    """The clock record a line carries: the median SM clock and the throttle reasons seen
    inside the timed window (plus a second of margin), from nvidia-smi's CSV rows as written
    with --format=csv,noheader,nounits."""
    sys.path.insert(0, ROOT)
    import time
    import bench
    t0 = time.mktime(time.strptime("2026/12/03 12:00:00", "%Y/%m/%d %H:%M:%S"))
    rows = [
        # before the window: a thermal slowdown that must not be reported
        "2026/12/03 11:59:50.100, 1200, 1965, 900.0, 0x20, Not Active, Not Active, Active, Not Active",
        "2026/12/03 12:00:00.100, 1965, 1965, 700.5, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/03 12:00:01.100, 1890, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/03 12:00:02.100, 1965, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "2026/12/03 12:00:30.100, 1000, 1965, 300.0, 0x8, Active, Not Active, Not Active, Not Active",
    ]
    s = bench.ClockSampler(None)
    s.file.write("\n".join(rows) + "\n")
    s.proc = _DoneProcess()
    rec = s.stop(t0, t0 + 2.0)
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]


def test_clock_record_without_nvidia_smi():
    sys.path.insert(0, ROOT)
    import bench
    s = bench.ClockSampler(None)
    s.proc = None
    rec = s.stop(0.0, 1.0)
    assert rec["samples"] == 0 and rec["sm_mhz"] is None
    os.unlink(s.file.name)
