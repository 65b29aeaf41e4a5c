#!/usr/bin/env python
"""Benchmark of the exact attention forward on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--sweep] [--rows]

Defaults: 5 warm-up steps, then 20 timed steps.  ``--sweep`` times the head-dim x length grid,
``--rows`` the strided, packed, FP8-with-two-lengths and d=64 entry points; ``--profile-case``
runs a few untimed calls of one entry point for an ncu capture.

A step is one call of the bf16 forward (``attn_fwd``) on the headline workload, bf16 B=2 H=16
N=8192 d=128 causal, inputs iid N(0,1) (seed 0 + rank), already resident in device memory.
``value`` is attention TFLOP/s with FLOPs = 4*B*H*N^2*d, halved for causal (diagonal-tile
work is not credited), summed over ranks and divided by the slowest rank's time.  Each step
is timed with CUDA events on the launching stream; a 256 MiB buffer is written between steps
(outside the events) so that every step starts with a cold L2.

Extra keys: ``roofline`` (the kernel's TFLOP/s against the measured burst dense bf16 peak;
the fraction of the measured sustained peak is given beside it, with a flag when the clock
record shows the timed loop ran power-capped),
``cpu_baseline`` (the float64 oracle on this host's cores, on a bounded sample of the same
workload), ``e2e`` (the same metric through the C ABI with pinned host buffers, copies
included), ``clocks`` (nvidia-smi samples during the timed region), ``gpu_launches``,
``fp8`` (the Hadamard/E4M3 pre-kernel and the E4M3 forward on their own workload, the FP8
roofline against an E4M3 cuBLAS GEMM measured in the same run, and the bf16 kernel on the same
shape), ``bwd``, ``varlen``, ``ring_merge`` and ``sweep`` (every head-dim x length point and the
B=4 H=16 N=2048 d=128 configuration, causal and not).

With N > 1 (under torchrun) every rank runs its own replica of the workload on its own GPU
(weak scaling, no collective on the data path; the process group only carries the timing
barrier and the max over ranks).  ``--impl reference`` runs the float64 oracle instead, on
the host cores, on a bounded sample per step (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn fwd TFLOP/s & % of B200 dense tensor peak (bf16 hd128 N=8K causal)"
WORKLOAD = dict(B=2, H=16, N=8192, d=128, causal=True)
FP8_WORKLOAD = dict(B=2, H=16, N=8192, d=128, causal=False, outlier_frac=1e-3)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def attn_flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


FWD_SOURCES = ("attn_fwd_kernel.cuh", "attn_fwd_sm100.cu", "attn_kernels.h", "sm100_ptx.cuh", "unit_table.cu")


def kernel_source_hash(names=FWD_SOURCES):
    """Hash of the sources a kernel is built from (the bf16 forward by default)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_attention_100_b200", "csrc")
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kind):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", f"{kind}.txt")
    try:
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("source_sha256_16", "").split(" ")[0] != kernel_source_hash():
            return None
        return float(fields["dram_bytes_per_launch_full_size"].split(" ")[0])
    except (OSError, KeyError, ValueError):
        return None


def measured_gemm_peaks(dev, n=8192, reps=10):
    """TFLOP/s of cuBLAS on this GPU in this run: a bf16 matmul and an E4M3 ``torch._scaled_mm``
    (tensorwise scales, bf16 out), n^3, best of ``reps`` after 3 warm-ups.  The E4M3 figure is
    the FP8 roofline's denominator (the driver's peaks file has no FP8 entry)."""
    import torch
    out = {}
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()  # column-major second operand
    one = torch.ones((), device=dev)
    ab, bb = a.to(torch.bfloat16), b.to(torch.bfloat16)
    for name, fn in (("e4m3_tflops", lambda: torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)),
                     ("bf16_tflops", lambda: ab @ bb)):
        try:
            for _ in range(3):
                fn()
            best = float("inf")
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                best = min(best, e0.elapsed_time(e1))
            out[name] = 2.0 * n ** 3 / (best * 1e-3) / 1e12
        except Exception as e:  # no FP8 GEMM in this torch build: the FP8 roofline falls back
            out[name + "_error"] = repr(e)
    return out


# ---------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid):
        self.file = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        self.proc = None
        self.uuid = device_uuid

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.t0 = time.time()

    def mark(self):
        return time.time()

    def stop(self, t_begin, t_end):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        self.file.flush()
        self.file.seek(0)
        rows = []
        for line in self.file.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.file.name)
        inside = [r for r in rows if t_begin - 1.0 <= r[0] <= t_end + 1.0] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, x in enumerate(r[3]) if x.lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in inside])), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


# ------------------------------------------------------------------------------ CPU oracle
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_head_sample(target_s=15.0, max_heads=8, seed=0):
    """Times the float64 oracle on whole heads of the headline workload (first heads of batch 0)."""
    from oracle import attention_ref
    from exact_attention_100_b200.inputs import normal_qkv
    w = WORKLOAD
    q, k, v = normal_qkv(1, max_heads, w["N"], w["d"], seed=seed)
    scale = 1.0 / math.sqrt(w["d"])
    t0 = time.perf_counter()
    attention_ref(q[0, :1], k[0, :1], v[0, :1], scale, w["causal"])
    t1 = time.perf_counter() - t0
    heads = int(max(1, min(max_heads, target_s // max(t1, 1e-3))))
    t0 = time.perf_counter()
    if heads > 1:
        attention_ref(q[0, 1:heads], k[0, 1:heads], v[0, 1:heads], scale, w["causal"])
    el = (time.perf_counter() - t0) + t1
    flops = attn_flops(1, heads, w["N"], w["d"], w["causal"])
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{heads} whole head(s) of the workload (batch 0, heads 0..{heads - 1}), float64 numpy, "
                      f"{el:.1f} s"}


def run_reference(args):
    """The float64 oracle as the reference arm: each step = the last R query rows of head 0."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import attention_ref
    from exact_attention_100_b200.inputs import normal_qkv
    w = WORKLOAD
    q, k, v = normal_qkv(1, 1, w["N"], w["d"], seed=0)
    scale = 1.0 / math.sqrt(w["d"])
    R = 32
    rows = range(w["N"] - R, w["N"])
    flops = sum(4.0 * w["d"] * (i + 1) for i in rows)  # causal: row i sees keys 0..i

    def step():
        for i in rows:  # the oracle on keys 0..i for each causal row
            attention_ref(q[0, 0, i:i + 1], k[0, 0, :i + 1], v[0, 0, :i + 1], scale, False)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    val = flops * args.steps / el / 1e12
    sample = f"last {R} query rows of head (0,0) per step, each row against its visible keys, float64 numpy"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "bf16 attention fwd B=2 H=16 N=8192 d=128 causal (oracle sample)", **WORKLOAD},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------------- rank aggregation
def max_over_ranks(x, world, device):
    """The largest ``x`` over the ranks of the default process group (the slowest rank's time);
    ``x`` itself with one rank.  ``device`` is where the reduction's tensor lives (the rank's GPU
    under NCCL, the CPU under gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world, flops_per_rank, ms_max):
    """Throughput of the whole job: every rank's work divided by the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


# ----------------------------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist
    import exact_attention_100_b200 as ea
    from exact_attention_100_b200.inputs import normal_qkv, hadamard_signs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def slowest(x):
        return max_over_ranks(x, world, dev)

    w = WORKLOAD
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    scale = 1.0 / math.sqrt(d)
    qn, kn, vn = normal_qkv(B, H, N, d, seed=rank)
    host = [torch.from_numpy(a).to(torch.bfloat16) for a in (qn, kn, vn)]
    q, k, v = (t.to(dev) for t in host)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    flops = attn_flops(B, H, N, d, causal)

    def step():
        ea.attn_fwd(q, k, v, o=o, lse=lse, scale=scale, causal=causal, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches0 = ea.attn_num_kernel_launches()
    barrier()
    torch.cuda.synchronize()
    t_begin = time.time()
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    t_end = time.time()
    launches = ea.attn_num_kernel_launches() - launches0
    ms = float(np.mean([s.elapsed_time(e) for s, e in zip(starts, ends)]))
    clocks = sampler.stop(t_begin, t_end) if sampler else None
    assert ea.attn_device_status() == ea.ATTN_OK
    ms_max = slowest(ms)
    value = whole_job_tflops(world, flops, ms_max)

    # e2e: pinned host inputs -> device -> attn_fwd -> O and LSE back to pinned host memory, every
    # step.  Two buffer slots and three streams: the host-to-device copy of step i+1 and the
    # device-to-host copy of step i-1 overlap the attention of step i (PCIe carries both
    # directions at once), as a pipeline feeding the library from host memory would run.
    pin_in = [t.pin_memory() for t in host]
    slots = []
    for _ in range(2):
        slots.append({"in": [torch.empty_like(t) for t in (q, k, v)], "o": torch.empty_like(o),
                      "lse": torch.empty_like(lse), "pin_o": torch.empty(o.shape, dtype=o.dtype).pin_memory(),
                      "pin_l": torch.empty(lse.shape, dtype=lse.dtype).pin_memory(),
                      "ev_in": torch.cuda.Event(), "ev_fwd": torch.cuda.Event(), "ev_out": torch.cuda.Event(),
                      "used": False})
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step(i):
        sl = slots[i % 2]
        with torch.cuda.stream(s_in):
            if sl["used"]:
                s_in.wait_event(sl["ev_fwd"])  # the slot's inputs are free once its last attention ran
            for dst, src in zip(sl["in"], pin_in):
                dst.copy_(src, non_blocking=True)
            sl["ev_in"].record(s_in)
        stream.wait_event(sl["ev_in"])
        if sl["used"]:
            stream.wait_event(sl["ev_out"])  # ... and its outputs once they reached the host
        ea.attn_fwd(*sl["in"], o=sl["o"], lse=sl["lse"], scale=scale, causal=causal, stream=stream)
        sl["ev_fwd"].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(sl["ev_fwd"])
            sl["pin_o"].copy_(sl["o"], non_blocking=True)
            sl["pin_l"].copy_(sl["lse"], non_blocking=True)
            sl["ev_out"].record(s_out)
        sl["used"] = True

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(s_in)
    stream.wait_event(ev0)
    s_out.wait_event(ev0)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_event(slots[(e2e_steps - 1) % 2]["ev_out"])
    stream.wait_event(slots[e2e_steps % 2]["ev_out"])
    ev1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = slowest(ev0.elapsed_time(ev1) / e2e_steps)
    pin_o, pin_l = slots[0]["pin_o"], slots[0]["pin_l"]
    h2d = sum(t.numel() * t.element_size() for t in pin_in)
    d2h = pin_o.numel() * pin_o.element_size() + pin_l.numel() * pin_l.element_size()

    fp8 = fp8_section(args, dev, rank) if not args.no_fp8 else None
    bwd = bwd_section(args, dev, rank) if not args.no_bwd else None
    varlen = varlen_section(args, dev, rank) if not args.no_varlen else None
    ring = ring_section(args, dev, rank) if not args.no_ring else None
    sweep = sweep_section(args, dev, uuid) if not args.no_sweep else None
    barrier()
    if rank == 0:
        peaks = load_peaks()
        burst = float(peaks["bf16_tflops"])
        sustained = float(peaks["bf16_tflops_sustained"]) if "bf16_tflops_sustained" in peaks else None
        # The primary denominator is the burst GEMM rate (the kernel is timed alone); a loop long
        # enough for the 1 kW cap to pull the SM clock down (sw_power_cap active, median clock
        # below 95% of max) is flagged, and its fraction of the sustained rate is given beside it.
        power_limited = bool(sustained and clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz")
                             and "sw_power_cap" in (clocks.get("reasons") or [])
                             and clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"])
        peak = burst
        achieved = flops / (ms * 1e-3) / 1e12
        traffic = profiled_traffic("attn_fwd_bf16_d128_n8192_causal")
        cpu = oracle_head_sample(target_s=args.cpu_seconds) if not args.no_cpu_baseline else None
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "bf16 attention fwd B=2 H=16 N=8192 d=128 causal (headline)",
                       "B": B, "H": H, "N": N, "d": d, "causal": causal, "o_dtype": "bf16", "lse": True,
                       "inputs": "iid N(0,1) rounded to bf16, seed 0 + rank, resident in HBM",
                       "l2": "256 MiB buffer written between timed steps (outside the events); inputs 192 MiB",
                       "parallelism": f"replicas x{world}: one full workload per GPU, no collective"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peaks['source']} bf16_tflops (burst, cuBLAS 8192^3) "
                                        f"-- fraction is of {peaks['source']}",
                         "power_capped_loop": power_limited,
                         "frac_of_measured_burst": achieved / burst,
                         "frac_of_measured_sustained": achieved / sustained if sustained else None,
                         "frac_of_datasheet_2250": achieved / 2250.0},
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_tflops(world, flops, e2e_ms), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "path": "pinned host -> H2D copies -> attn_fwd (C ABI) -> D2H O, LSE",
                    "overlap": "two buffer slots, three streams: H2D of step i+1 and D2H of step i-1 overlap the "
                               "attention of step i"},
            "gpu_launches": launches,
            "clocks": clocks,
        }
        if fp8 is not None:
            line["fp8"] = fp8
        if bwd is not None:
            line["bwd"] = bwd
        if varlen is not None:
            line["varlen"] = varlen
        if ring is not None:
            line["ring_merge"] = ring
        if sweep is not None:
            line["sweep"] = sweep
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def fp8_section(args, dev, rank):
    """Times the Hadamard/E4M3 pre-kernel (3 tensors) and the E4M3 forward on the FP8 workload."""
    import torch
    import exact_attention_100_b200 as ea
    from exact_attention_100_b200.inputs import normal_qkv, hadamard_signs
    w = FP8_WORKLOAD
    B, H, N, d = w["B"], w["H"], w["N"], w["d"]
    qn, kn, vn = normal_qkv(B, H, N, d, seed=rank, outlier_frac=w["outlier_frac"])
    q, k, v = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
    signs = torch.from_numpy(hadamard_signs(d)).to(dev)
    nb = (N + 127) // 128
    x8 = [torch.empty(q.shape, dtype=torch.uint8, device=dev) for _ in range(3)]
    sc = [torch.empty((B, H, nb), dtype=torch.float32, device=dev) for _ in range(3)]
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    outs = (x8[0], x8[1], x8[2], sc[0], sc[1], sc[2])

    def pre():  # one launch for the three tensors (Q, K transformed; V not)
        ea.attn_hadamard_quant_qkv(q, k, v, signs, outs=outs, stream=stream)

    steps = max(3, min(args.steps, 50))
    for _ in range(3):
        pre()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        pre()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    pre_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    elems = 3 * q.numel()
    pre_bytes = elems * 3 + 3 * B * H * nb * 4  # 2 B read + 1 B written per element, plus scales
    peaks = load_peaks()
    gbs = pre_bytes / (pre_ms * 1e-3) / 1e9
    out = {"workload": "B=2 H=16 N=8192 d=128 non-causal, 0.1% N(0,10^2) outliers, seeded signs",
           "prekernel": {"ms_3_tensors": pre_ms, "achieved_gbs": gbs, "peak_gbs": float(peaks["hbm_gbs"]),
                         "frac": gbs / float(peaks["hbm_gbs"]), "bound": "hbm",
                         "bytes_per_call": pre_bytes, "peak_source": peaks["source"]}}

    # the same launch with the rotary embedding of Q and K fused in front of the transform
    from exact_attention_100_b200.inputs import rope_tables
    cos_n, sin_n = rope_tables(N, d)  # [N, d/2]; the kernel takes them frequency-major
    cos, sin = (torch.from_numpy(np.ascontiguousarray(t.T)).to(dev) for t in (cos_n, sin_n))

    def pre_rope():
        ea.attn_rope_hadamard_quant_qkv(q, k, v, signs, cos, sin, outs=outs, stream=stream)

    for _ in range(3):
        pre_rope()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        pre_rope()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    rope_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    rope_bytes = pre_bytes + 2 * N * (d // 2) * 4  # plus the cos and sin tables, read once from HBM
    rgbs = rope_bytes / (rope_ms * 1e-3) / 1e9
    out["prekernel_rope"] = {"ms_3_tensors": rope_ms, "achieved_gbs": rgbs, "peak_gbs": float(peaks["hbm_gbs"]),
                             "frac": rgbs / float(peaks["hbm_gbs"]), "bound": "hbm", "bytes_per_call": rope_bytes,
                             "vs_unrotated": rope_ms / pre_ms, "peak_source": peaks["source"],
                             "note": "Q and K rotated (frequency-major tables [64, 8192] float32, L2-resident "
                                     "after the first read), then H D and E4M3; V quantised as it is"}

    # the same launch reading Q, K, V as head views of one fused [B, N, 3, H, d] projection
    fused = torch.empty((B, N, 3, H, d), dtype=torch.bfloat16, device=dev)
    views = [fused[:, :, j].transpose(1, 2) for j in range(3)]
    for view, x in zip(views, (q, k, v)):
        view.copy_(x)

    def pre_strided():
        ea.attn_hadamard_quant_qkv_strided(views[0], views[1], views[2], signs, outs=outs, stream=stream)

    for _ in range(3):
        pre_strided()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        pre_strided()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    st_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    sgbs = pre_bytes / (st_ms * 1e-3) / 1e9
    out["prekernel_strided"] = {"ms_3_tensors": st_ms, "achieved_gbs": sgbs, "frac": sgbs / float(peaks["hbm_gbs"]),
                                "vs_contiguous": st_ms / pre_ms, "bytes_per_call": pre_bytes,
                                "note": "Q, K, V read as head views of one fused [B, N, 3, H, d] bf16 buffer "
                                        "(attn_hadamard_quant_qkv_strided); contiguous E4M3 outputs"}
    del fused, views
    try:
        o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)

        def fwd8():
            ea.attn_fwd_fp8(x8[0], x8[1], x8[2], sc[0], sc[1], sc[2], o=o, lse=lse, causal=w["causal"], stream=stream)

        for _ in range(3):
            fwd8()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(float(i))
            evs[i][0].record(stream)
            fwd8()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        ms8 = float(np.mean([a.elapsed_time(b) for a, b in evs]))
        fl = attn_flops(B, H, N, d, w["causal"])
        gemm = measured_gemm_peaks(dev)
        if "e4m3_tflops" in gemm:
            fp8_peak = gemm["e4m3_tflops"]
            src = "measured in this run: torch._scaled_mm E4M3 8192^3, tensorwise scales, best of 10"
        else:
            fp8_peak = 2.0 * float(peaks["bf16_tflops"])
            src = f"2 x {peaks['source']} bf16_tflops (no FP8 GEMM measurement: {gemm.get('e4m3_tflops_error')})"
        tf8 = fl / (ms8 * 1e-3) / 1e12
        out["forward"] = {"ms": ms8, "achieved_tflops": tf8, "peak_tflops": fp8_peak, "frac": tf8 / fp8_peak,
                          "peak_source": src, "gemm_peaks_this_run": gemm}
        # the bf16 kernel on the same shape and inputs (unquantised), for the FP8 speed-up
        ob = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)

        def fwd16():
            ea.attn_fwd(q, k, v, o=ob, lse=lse, causal=w["causal"], stream=stream)

        for _ in range(3):
            fwd16()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(float(i))
            evs[i][0].record(stream)
            fwd16()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        ms16 = float(np.mean([a.elapsed_time(b) for a, b in evs]))
        out["forward"]["bf16_same_shape"] = {"ms": ms16, "achieved_tflops": fl / (ms16 * 1e-3) / 1e12,
                                             "fp8_speedup": ms16 / ms8}
        out["forward_d256"] = fp8_other_d_section(dev, rank, steps, flush, fp8_peak, d=256)
        out["forward_d64"] = fp8_other_d_section(dev, rank, steps, flush, fp8_peak, d=64)
    except Exception as e:  # the E4M3 forward reports unsupported until it is built
        out["forward"] = {"unavailable": str(e)}
    return out


def fp8_other_d_section(dev, rank, steps, flush, fp8_peak, d=256):
    """The E4M3 forward at another head dim on the same token count (B=2 H=2048/d N=8192,
    non-causal, the outlier recipe, Hadamard on Q and K), and the bf16 kernel on the same
    unquantised inputs."""
    import torch
    import exact_attention_100_b200 as ea
    from exact_attention_100_b200.inputs import normal_qkv, hadamard_signs
    B, H, N = 2, 2048 // d, 8192
    qn, kn, vn = normal_qkv(B, H, N, d, seed=rank, outlier_frac=1e-3)
    q, k, v = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
    signs = torch.from_numpy(hadamard_signs(d)).to(dev)
    q8 = ea.attn_hadamard_quant_qkv(q, k, v, signs)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(3):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(float(i))
            evs[i][0].record(stream)
            fn()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in evs]))

    ms_pre = timed(lambda: ea.attn_hadamard_quant_qkv(q, k, v, signs, outs=q8, stream=stream))
    ms8 = timed(lambda: ea.attn_fwd_fp8(*q8, o=o, lse=lse, causal=False, stream=stream))
    ms16 = timed(lambda: ea.attn_fwd(q, k, v, o=o, lse=lse, causal=False, stream=stream))
    fl = attn_flops(B, H, N, d, False)
    assert ea.attn_device_status() == ea.ATTN_OK
    peaks = load_peaks()
    pre_bytes = 3 * q.numel() * 3 + 3 * B * H * ((N + 127) // 128) * 4  # 2 B read + 1 B written, scales
    pre_gbs = pre_bytes / (ms_pre * 1e-3) / 1e9
    return {"workload": f"B=2 H={H} N=8192 d={d} non-causal, 0.1% N(0,10^2) outliers, seeded signs", "ms": ms8,
            "achieved_tflops": fl / (ms8 * 1e-3) / 1e12, "frac": fl / (ms8 * 1e-3) / 1e12 / fp8_peak,
            "bf16_same_shape_ms": ms16, "fp8_speedup": ms16 / ms8,
            "prekernel": {"ms_3_tensors": ms_pre, "achieved_gbs": pre_gbs, "frac": pre_gbs / float(peaks["hbm_gbs"]),
                          "bound": "hbm", "bytes_per_call": pre_bytes, "peak_source": peaks["source"]}}


def ring_section(args, dev, rank):
    """Times the partial-result merge of the ring attention (attn_merge_partials) on the
    headline's rows: float32 accumulator [2, 16, 8192, 128], bf16 part; HBM-bound."""
    import torch
    import exact_attention_100_b200 as ea
    B, H, N, d = 2, 16, 8192, 128
    g = torch.Generator(device=dev).manual_seed(17 + rank)
    acc_o = torch.randn(B, H, N, d, device=dev, generator=g)
    acc_l = torch.randn(B, H, N, device=dev, generator=g)
    part_o = torch.randn(B, H, N, d, device=dev, generator=g).to(torch.bfloat16)
    part_l = torch.randn(B, H, N, device=dev, generator=g)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for _ in range(3):
        ea.attn_merge_partials(acc_o, acc_l, part_o, part_l, stream=stream)
    steps = max(3, min(args.steps, 50))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        ea.attn_merge_partials(acc_o, acc_l, part_o, part_l, stream=stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    rows = B * H * N
    nbytes = rows * d * (4 + 2 + 4) + rows * 4 * 3  # acc read + part read + acc written; three LSE rows
    peaks = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": "merge of a bf16 partial (O, LSE) into a float32 accumulator, rows [2, 16, 8192], d=128",
            "ms": ms, "achieved_gbs": gbs, "peak_gbs": float(peaks["hbm_gbs"]), "frac": gbs / float(peaks["hbm_gbs"]),
            "bound": "hbm", "bytes_per_call": nbytes, "peak_source": peaks["source"]}


VARLEN_WORKLOAD = dict(total=16384, lo=512, hi=4096, H=16, d=128, causal=True, seed=11)


def varlen_lengths(total, lo, hi, seed):
    """Sequence lengths drawn uniformly from [lo, hi] until they hold `total` tokens (the last one
    cut to fit)."""
    from exact_attention_100_b200.inputs import uniform_lengths
    pool = [int(x) for x in uniform_lengths(4 * total // lo + 1, lo, hi, seed=seed)]
    out, acc = [], 0
    for n in pool:
        n = min(n, total - acc)
        out.append(n)
        acc += n
        if acc == total:
            break
    return out


def varlen_section(args, dev, rank):
    """Times attn_fwd_varlen on a packed batch holding as many query tokens as the headline
    (2 x 8192), in sequences of 512..4096 tokens; FLOPs are counted per sequence."""
    import torch
    import exact_attention_100_b200 as ea
    from exact_attention_100_b200.inputs import normal_qkv_packed
    w = VARLEN_WORKLOAD
    lens = varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
    H, d, causal = w["H"], w["d"], w["causal"]
    qn, kn, vn, cq, ck = normal_qkv_packed(lens, lens, H, d, seed=w["seed"] + rank)
    q, k, v = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
    cu_q, cu_k = (torch.from_numpy(a).to(dev) for a in (cq, ck))
    stream = torch.cuda.current_stream()
    o = torch.empty_like(q)
    lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step():
        ea.attn_fwd_varlen(q, k, v, cu_q, cu_k, max(lens), o=o, lse=lse, causal=causal, stream=stream)

    for _ in range(3):
        step()
    steps = max(3, min(args.steps, 50))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    flops = sum(attn_flops(1, H, n, d, causal) for n in lens)
    peaks = load_peaks()
    tf = flops / (ms * 1e-3) / 1e12
    # the backward of the same packed batch (bf16 gradients, dO iid N(0,1) by torch)
    dout = torch.randn(q.shape, generator=torch.Generator(device=dev).manual_seed(3), device=dev).to(torch.bfloat16)
    g = [torch.empty_like(q) for _ in range(3)]
    ws = torch.empty(ea.attn_bwd_workspace_bytes(len(lens), H, max(lens)) // 4, dtype=torch.float32, device=dev)

    def bstep():
        ea.attn_bwd_varlen(q, k, v, o, lse, dout, cu_q, cu_k, max(lens), max(lens), dq=g[0], dk=g[1], dv=g[2],
                           workspace=ws, causal=causal, stream=stream)

    for _ in range(3):
        bstep()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        bstep()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    bms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    btf = 2.5 * flops / (bms * 1e-3) / 1e12
    # the same backward with dS kept in the workspace (attn_bwd_varlen_ds)
    ws_ds = torch.empty(ea.attn_bwd_varlen_ds_workspace_bytes(len(lens), H, max(lens), max(lens)), dtype=torch.uint8,
                        device=dev)

    def dsstep():
        ea.attn_bwd_varlen_ds(q, k, v, o, lse, dout, cu_q, cu_k, max(lens), max(lens), dq=g[0], dk=g[1], dv=g[2],
                              workspace=ws_ds, causal=causal, stream=stream)

    for _ in range(3):
        dsstep()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        dsstep()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    dms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    dtf = 2.5 * flops / (dms * 1e-3) / 1e12
    del ws_ds
    # the E4M3 forward of the same packed batch: codes and per-sequence block scales from the
    # packed pre-kernel (Q, K through H D), then attn_fwd_fp8_varlen
    from exact_attention_100_b200.inputs import hadamard_signs
    signs = torch.from_numpy(hadamard_signs(d)).to(dev)
    q8s = ea.attn_hadamard_quant_qkv_varlen(q, k, v, signs, cu_q, cu_k, max(lens), max(lens))
    o8 = torch.empty_like(q)

    def fstep():
        ea.attn_fwd_fp8_varlen(*q8s, cu_q, cu_k, max(lens), max(lens), o=o8, lse=lse, causal=causal, stream=stream)

    for _ in range(3):
        fstep()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        fstep()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    fms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    ftf = flops / (fms * 1e-3) / 1e12
    return {"workload": f"bf16 packed varlen fwd, {len(lens)} sequences of {w['lo']}..{w['hi']} tokens "
                        f"(total {w['total']}), H={H} d={d} causal",
            "lengths": lens, "ms": ms, "achieved_tflops": tf, "peak_tflops": float(peaks["bf16_tflops"]),
            "frac": tf / float(peaks["bf16_tflops"]), "bound": "tensor", "flops_per_call": flops,
            "flops_note": "sum over sequences of 4 H d N^2 / 2 (causal), as the headline counts",
            "peak_source": peaks["source"],
            "bwd": {"entry_point": "attn_bwd_varlen_ds", "ms": dms, "achieved_tflops": dtf,
                    "frac": dtf / float(peaks["bf16_tflops"]),
                    "flops_note": "2.5 x the forward count (five products), bf16 gradients, 3 launches",
                    "recompute": {"entry_point": "attn_bwd_varlen", "ms": bms, "achieved_tflops": btf,
                                  "frac": btf / float(peaks["bf16_tflops"])}},
            "fp8_fwd": {"ms": fms, "achieved_tflops": ftf, "vs_bf16": ms / fms,
                        "note": "attn_fwd_fp8_varlen on the same batch (E4M3 codes and per-sequence "
                                "128-row block scales from attn_hadamard_quant_qkv_varlen; the "
                                "pre-kernel is not in the timed region), bf16 O"}}


def bwd_section(args, dev, rank):
    """Times the backward on the headline workload (device-resident inputs, bf16 gradients):
    attn_bwd_ds (dS kept in a 2.2 GB workspace, five products) as the line's figure, and
    attn_bwd (dQ recomputes S and dP, a 2 MB workspace) beside it."""
    import torch
    import exact_attention_100_b200 as ea
    from exact_attention_100_b200.inputs import normal_qkv, normal_dout
    w = WORKLOAD
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    qn, kn, vn = normal_qkv(B, H, N, d, seed=rank)
    q, k, v = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
    do = torch.from_numpy(normal_dout(B, H, N, d, seed=7 + rank)).to(torch.bfloat16).to(dev)
    stream = torch.cuda.current_stream()
    o, lse = ea.attn_fwd(q, k, v, causal=causal, stream=stream)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    steps = max(3, min(args.steps, 50))

    def timed(step):
        for _ in range(3):
            step()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(float(i))
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        assert ea.attn_device_status() == ea.ATTN_OK
        return float(np.mean([a.elapsed_time(b) for a, b in evs]))

    ws = torch.empty(ea.attn_bwd_workspace_bytes(B, H, N) // 4, dtype=torch.float32, device=dev)
    ms_rc = timed(lambda: ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, causal=causal, stream=stream))
    ws_ds = torch.empty(ea.attn_bwd_ds_workspace_bytes(B, H, N, causal), dtype=torch.uint8, device=dev)
    ms = timed(lambda: ea.attn_bwd_ds(q, k, v, o, lse, do, dq, dk, dv, ws_ds, causal=causal, stream=stream))
    flops = 2.5 * attn_flops(B, H, N, d, causal)  # dV, dP, S, dK, dQ: five N x N x d products
    peaks = load_peaks()
    tf, tf_rc = flops / (ms * 1e-3) / 1e12, flops / (ms_rc * 1e-3) / 1e12
    out = {"workload": "bf16 attention bwd B=2 H=16 N=8192 d=128 causal (dQ, dK, dV from O, LSE, dO)",
           "entry_point": "attn_bwd_ds", "ms": ms, "achieved_tflops": tf,
           "peak_tflops": float(peaks["bf16_tflops"]), "frac": tf / float(peaks["bf16_tflops"]), "bound": "tensor",
           "flops_per_call": flops, "flops_note": "algorithmic 2.5 x forward (five products)",
           "workspace_bytes": int(ws_ds.numel()), "launches_per_call": 3, "peak_source": peaks["source"],
           "note": "attn_bwd_ds: the dK/dV kernel stores each bf16 dS tile, a third kernel streams them with K "
                   "through the tensor cores for dQ (no recomputation)",
           "recompute": {"entry_point": "attn_bwd", "ms": ms_rc, "achieved_tflops": tf_rc,
                         "frac": tf_rc / float(peaks["bf16_tflops"]), "workspace_bytes": int(ws.numel() * 4),
                         "note": "dQ recomputes S and dP: seven products on the tensor cores"},
           "ds_vs_recompute": ms_rc / ms}
    del ws_ds
    return out


SWEEP_DS = (64, 128, 256)
SWEEP_NS = (512, 1024, 2048, 4096, 8192, 16384)


def sweep_section(args, dev, uuid=None):
    """The head-dim x length sweep (16384 tokens per head-batch: B = 16384/N, H = 2048/d, causal and
    not) and the B=4 H=16 N=2048 d=128 configuration, each timed like the headline (3 warm-ups,
    then the mean of 10 calls with a cold L2).  Inputs are iid N(0,1) drawn by torch on the device
    (the timing does not depend on the generator); parity at these sizes is in the GPU tests."""
    import torch
    import exact_attention_100_b200 as ea
    peaks = load_peaks()
    burst = float(peaks["bf16_tflops"])
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    g = torch.Generator(device=dev).manual_seed(1)
    points = [("C4", d, N, 16384 // N, 2048 // d) for d in SWEEP_DS for N in SWEEP_NS] + [("C2", 128, 2048, 4, 16)]
    out = []
    sampler = ClockSampler(uuid)
    sampler.start()
    t_begin = time.time()
    for (cfg, d, N, B, H) in points:
        q, k, v = (torch.randn(B, H, N, d, device=dev, generator=g).to(torch.bfloat16) for _ in range(3))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        for causal in (False, True):
            for _ in range(3):
                ea.attn_fwd(q, k, v, o=o, lse=lse, causal=causal, stream=stream)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
            for i in range(10):
                flush.fill_(float(i))
                evs[i][0].record(stream)
                ea.attn_fwd(q, k, v, o=o, lse=lse, causal=causal, stream=stream)
                evs[i][1].record(stream)
            torch.cuda.synchronize()
            ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
            tf = attn_flops(B, H, N, d, causal) / (ms * 1e-3) / 1e12
            out.append({"config": cfg, "d": d, "N": N, "B": B, "H": H,
                        "causal": causal, "ms": round(ms, 5), "tflops": round(tf, 1), "frac": round(tf / burst, 4)})
        del q, k, v, o, lse
    t_end = time.time()
    assert ea.attn_device_status() == ea.ATTN_OK
    return {"points": out, "peak_tflops": burst, "peak_source": peaks["source"],
            "timing": "3 warm-ups, mean of 10 calls, 256 MiB buffer written between calls",
            "clocks": sampler.stop(t_begin, t_end),
            "clocks_note": "the whole sweep runs back to back after the other sections; a median SM clock below "
                           "the maximum with sw_power_cap means its longer points ran power-capped"}


def run_sweep(args):
    """Head-dim / length sweep at 16K tokens per head-batch: one JSON line per point (rank 0)."""
    import torch
    import exact_attention_100_b200 as ea
    from exact_attention_100_b200.inputs import normal_qkv
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for d in (64, 128, 256):
        for N in (512, 1024, 2048, 4096, 8192, 16384):
            B, H = 16384 // N, 2048 // d
            qn, kn, vn = normal_qkv(B, H, N, d, seed=0)
            q, k, v = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
            o = torch.empty_like(q)
            lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
            for causal in (False, True):
                for _ in range(3):
                    ea.attn_fwd(q, k, v, o=o, lse=lse, causal=causal, stream=stream)
                n = max(5, min(args.steps, 30))
                evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
                for i in range(n):
                    flush.fill_(float(i))
                    evs[i][0].record(stream)
                    ea.attn_fwd(q, k, v, o=o, lse=lse, causal=causal, stream=stream)
                    evs[i][1].record(stream)
                torch.cuda.synchronize()
                ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
                tf = attn_flops(B, H, N, d, causal) / (ms * 1e-3) / 1e12
                print(json.dumps({"sweep": True, "d": d, "N": N, "B": B, "H": H, "causal": causal, "ms": ms,
                                  "tflops": tf, "frac_of_measured_bf16": tf / float(peaks["bf16_tflops"])}),
                      flush=True)


def run_rows(args):
    """Timings of the entry points the headline line does not cover, one JSON line: the strided
    forward and backward on the headline in sequence-major memory (against the contiguous entry
    points in the same run), the packed backward on the packed workload, the E4M3 forward with
    two lengths, and the d=64 backward.  20 steps each after 3 warm-ups, L2 flushed between."""
    import torch
    import exact_attention_100_b200 as ea
    from exact_attention_100_b200.inputs import hadamard_signs, normal_qkv_lengths, normal_qkv_packed
    dev = torch.device("cuda", 0)
    torch.manual_seed(0)
    flush = torch.empty(256 * 1024 * 1024 // 4, device=dev)
    steps = max(3, min(args.steps, 50))

    def timed(fn):
        for _ in range(3):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(float(i))
            evs[i][0].record()
            fn()
            evs[i][1].record()
        torch.cuda.synchronize()
        if ea.attn_device_status() != ea.ATTN_OK:
            raise SystemExit("device status set")
        return float(np.mean([a.elapsed_time(b) for a, b in evs]))

    peak = float(load_peaks()["bf16_tflops"])
    out = {}
    B, H, N, d = 2, 16, 8192, 128
    q, k, v = (torch.randn(B, N, H, d, device=dev).to(torch.bfloat16).transpose(1, 2) for _ in range(3))
    qc, kc, vc = (x.contiguous() for x in (q, k, v))
    fl = attn_flops(B, H, N, d, True)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=dev)
    ms_s = timed(lambda: ea.attn_fwd_strided(q, k, v, o=o, lse=lse, causal=True))
    ms_c = timed(lambda: ea.attn_fwd(qc, kc, vc, causal=True))
    out["fwd_strided_seq_major"] = {"ms": ms_s, "tflops": fl / ms_s / 1e9, "frac": fl / ms_s / 1e9 / peak,
                                    "contiguous_ms": ms_c, "contiguous_tflops": fl / ms_c / 1e9}
    do = torch.randn_like(qc)
    dos = do.transpose(1, 2).contiguous().transpose(1, 2)
    oc, lc = ea.attn_fwd(qc, kc, vc, causal=True)
    os_ = oc.transpose(1, 2).contiguous().transpose(1, 2)
    ws = torch.empty(ea.attn_bwd_workspace_bytes(B, H, N) // 4, device=dev)
    g = [torch.empty_like(q) for _ in range(3)]
    gc = [torch.empty_like(qc) for _ in range(3)]
    ms_bs = timed(lambda: ea.attn_bwd_strided(q, k, v, os_, lc, dos, dq=g[0], dk=g[1], dv=g[2], workspace=ws,
                                              causal=True))
    ms_bc = timed(lambda: ea.attn_bwd(qc, kc, vc, oc, lc, do, dq=gc[0], dk=gc[1], dv=gc[2], workspace=ws, causal=True))
    out["bwd_strided_seq_major"] = {"ms": ms_bs, "tflops": 2.5 * fl / ms_bs / 1e9, "frac": 2.5 * fl / ms_bs / 1e9 / peak,
                                    "contiguous_ms": ms_bc, "contiguous_tflops": 2.5 * fl / ms_bc / 1e9}
    w = VARLEN_WORKLOAD
    lens = varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
    qn, kn, vn, cq, ck = normal_qkv_packed(lens, lens, w["H"], w["d"], seed=w["seed"])
    pq, pk, pv = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
    tcq, tck = torch.from_numpy(cq).to(dev), torch.from_numpy(ck).to(dev)
    po, pl = ea.attn_fwd_varlen(pq, pk, pv, tcq, tck, max(lens), causal=True)
    pdo = torch.randn_like(pq)
    pws = torch.empty(ea.attn_bwd_workspace_bytes(len(lens), w["H"], max(lens)) // 4, device=dev)
    pg = [torch.empty_like(pq) for _ in range(3)]
    vfl = sum(attn_flops(1, w["H"], n, w["d"], True) for n in lens)
    ms_pv = timed(lambda: ea.attn_bwd_varlen(pq, pk, pv, po, pl, pdo, tcq, tck, max(lens), max(lens), dq=pg[0], dk=pg[1],
                                             dv=pg[2], workspace=pws, causal=True))
    out["bwd_varlen"] = {"ms": ms_pv, "tflops": 2.5 * vfl / ms_pv / 1e9, "frac": 2.5 * vfl / ms_pv / 1e9 / peak,
                         "lengths": lens}
    qn, kn, vn = normal_qkv_lengths(2, 16, 4096, 8192, 128, seed=3)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
    sg = torch.from_numpy(hadamard_signs(128)).to(dev)
    q8, qs = ea.attn_hadamard_quant(tq, sg)
    k8, ks = ea.attn_hadamard_quant(tk, sg)
    v8, vs = ea.attn_hadamard_quant(tv, None)
    o8 = torch.empty(2, 16, 4096, 128, dtype=torch.bfloat16, device=dev)
    l8 = torch.empty(2, 16, 4096, device=dev)
    ms8 = timed(lambda: ea.attn_fwd_fp8_qk(q8, k8, v8, qs, ks, vs, o=o8, lse=l8, causal=False))
    fl8 = 4.0 * 2 * 16 * 4096 * 8192 * 128
    out["fp8_qk"] = {"ms": ms8, "tflops": fl8 / ms8 / 1e9, "frac": fl8 / ms8 / 1e9 / (2 * peak),
                     "workload": "B=2 H=16 Nq=4096 Nk=8192 d=128 non-causal, peak 2 x bf16"}
    q6, k6, v6 = (torch.randn(2, 32, 8192, 64, device=dev).to(torch.bfloat16) for _ in range(3))
    o6, l6 = ea.attn_fwd(q6, k6, v6, causal=True)
    do6 = torch.randn_like(q6)
    ws6 = torch.empty(ea.attn_bwd_workspace_bytes(2, 32, 8192) // 4, device=dev)
    g6 = [torch.empty_like(q6) for _ in range(3)]
    ms6 = timed(lambda: ea.attn_bwd(q6, k6, v6, o6, l6, do6, dq=g6[0], dk=g6[1], dv=g6[2], workspace=ws6, causal=True))
    fl6 = 2.5 * attn_flops(2, 32, 8192, 64, True)
    out["bwd_d64"] = {"ms": ms6, "tflops": fl6 / ms6 / 1e9, "frac": fl6 / ms6 / 1e9 / peak,
                      "workload": "B=2 H=32 N=8192 d=64 causal"}
    print(json.dumps({"rows": out, "peak_tflops": peak, "steps": steps}), flush=True)


def run_profile_case(args):
    """A few untimed calls of one entry point on a small case, for an ncu capture (no JSON line)."""
    import torch
    import exact_attention_100_b200 as ea
    from exact_attention_100_b200.inputs import hadamard_signs
    B, H, N, d, causal = args.shape
    dev = torch.device("cuda", 0)
    torch.manual_seed(0)
    q, k, v = (torch.randn(B, H, N, d, device=dev).to(torch.bfloat16) for _ in range(3))
    signs = torch.from_numpy(hadamard_signs(d)).to(dev)
    if args.profile_case == "fwd":
        for _ in range(args.reps):
            ea.attn_fwd(q, k, v, causal=bool(causal))
    elif args.profile_case == "merge":
        acc_o = torch.randn(B, H, N, d, device=dev)
        acc_l = torch.randn(B, H, N, device=dev)
        part_o = torch.randn(B, H, N, d, device=dev).to(torch.bfloat16)
        part_l = torch.randn(B, H, N, device=dev)
        for _ in range(args.reps):
            ea.attn_merge_partials(acc_o, acc_l, part_o, part_l)
    elif args.profile_case == "hq_rope":
        from exact_attention_100_b200.inputs import rope_tables
        cos, sin = (torch.from_numpy(np.ascontiguousarray(t.T)).to(dev) for t in rope_tables(N, d))
        outs = None
        for _ in range(args.reps):
            outs = ea.attn_rope_hadamard_quant_qkv(q, k, v, signs, cos, sin, outs=outs)
    elif args.profile_case == "varlen":
        # the bench's packed workload (the shape's H and d; lengths from the packed recipe)
        from exact_attention_100_b200.inputs import normal_qkv_packed
        w = VARLEN_WORKLOAD
        lens = varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
        qn, kn, vn, cq, ck = normal_qkv_packed(lens, lens, H, d, seed=w["seed"])
        pq, pk, pv = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
        cu_q, cu_k = torch.from_numpy(cq).to(dev), torch.from_numpy(ck).to(dev)
        for _ in range(args.reps):
            ea.attn_fwd_varlen(pq, pk, pv, cu_q, cu_k, max(lens), causal=bool(causal))
    elif args.profile_case == "fp8_varlen":
        # the bench's packed batch through the packed pre-kernel and the packed E4M3 forward
        from exact_attention_100_b200.inputs import normal_qkv_packed
        w = VARLEN_WORKLOAD
        lens = varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
        qn, kn, vn, cq, ck = normal_qkv_packed(lens, lens, H, d, seed=w["seed"])
        pq, pk, pv = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
        cu_q, cu_k = torch.from_numpy(cq).to(dev), torch.from_numpy(ck).to(dev)
        outs = ea.attn_hadamard_quant_qkv_varlen(pq, pk, pv, signs, cu_q, cu_k, max(lens), max(lens))
        for _ in range(args.reps):
            ea.attn_fwd_fp8_varlen(*outs, cu_q, cu_k, max(lens), max(lens), causal=bool(causal))
    elif args.profile_case == "varlen_bwd_ds":
        # the bench's packed batch through the packed backward with dS kept
        from exact_attention_100_b200.inputs import normal_qkv_packed
        w = VARLEN_WORKLOAD
        lens = varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
        qn, kn, vn, cq, ck = normal_qkv_packed(lens, lens, H, d, seed=w["seed"])
        pq, pk, pv = (torch.from_numpy(a).to(torch.bfloat16).to(dev) for a in (qn, kn, vn))
        cu_q, cu_k = torch.from_numpy(cq).to(dev), torch.from_numpy(ck).to(dev)
        po, pl = ea.attn_fwd_varlen(pq, pk, pv, cu_q, cu_k, max(lens), causal=bool(causal))
        pdo = torch.randn_like(pq)
        for _ in range(args.reps):
            ea.attn_bwd_varlen_ds(pq, pk, pv, po, pl, pdo, cu_q, cu_k, max(lens), max(lens), causal=bool(causal))
    elif args.profile_case == "bwd":
        o, lse = ea.attn_fwd(q, k, v, causal=bool(causal))
        do = torch.randn_like(q)
        for _ in range(args.reps):
            ea.attn_bwd(q, k, v, o, lse, do, causal=bool(causal))
    elif args.profile_case == "bwd_ds":
        o, lse = ea.attn_fwd(q, k, v, causal=bool(causal))
        do = torch.randn_like(q)
        for _ in range(args.reps):
            ea.attn_bwd_ds(q, k, v, o, lse, do, causal=bool(causal))
    else:
        outs = None
        for _ in range(args.reps):
            outs = ea.attn_hadamard_quant_qkv(q, k, v, signs, outs=outs)
        if args.profile_case == "fwd_fp8":
            for _ in range(args.reps):
                ea.attn_fwd_fp8(*outs, causal=bool(causal))
    torch.cuda.synchronize()
    if ea.attn_device_status() != 0:
        raise SystemExit("device status set")
    print("ok", args.profile_case, B, H, N, d, causal, flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--rows", action="store_true",
                    help="time the entry points the headline line does not cover and exit")
    ap.add_argument("--no-fp8", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-varlen", action="store_true")
    ap.add_argument("--no-ring", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="leave the head-dim x length sweep out of the line")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile-case", choices=["fwd", "fwd_fp8", "hq_qkv", "hq_rope", "varlen", "fp8_varlen", "varlen_bwd_ds", "bwd", "bwd_ds",
                             "merge"], default=None,
                    help="run --reps untimed calls of one entry point (for an ncu capture) and exit")
    ap.add_argument("--shape", type=int, nargs=5, default=[2, 16, 8192, 128, 1], metavar=("B", "H", "N", "d", "CAUSAL"))
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    if args.profile_case is not None:
        run_profile_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    elif args.rows:
        run_rows(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
