"""The allocation-free entry point, attn_fwd_noalloc, against the float64 oracle and attn_fwd (GPU).

attn_fwd_noalloc is for callers that cannot let the library call cudaMalloc (runtimes that
own all device memory through their own pool, hosts with a fixed memory budget, loops that
must never reach an allocation that may synchronise the device): its scratch is a static
device array of the library.  Its results must meet the oracle's parity bars and match
attn_fwd within them, on two calls in a row (the second call finds the array holding the
first call's contents).  Its status word is read by attn_noalloc_status.  This file is
collected last on purpose.
"""

import ctypes
import json
import math
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build
from gpu_util import LSE_REL, O_MAX_ABS, O_MEAN_ABS, assert_within, compare_full, device_qkv

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _call_noalloc(q, k, v, o, lse, causal):
    B, H, N, d = q.shape
    od = ea.ATTN_FP32 if o.dtype == torch.float32 else ea.ATTN_BF16
    s = torch.cuda.current_stream()
    return ea.lib().attn_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), B, H, N, d, 1.0 / math.sqrt(d),
        int(causal), ea.ATTN_BF16, od, ctypes.c_void_p(s.cuda_stream))


@pytest.mark.parametrize("B,H,N,d,causal,o_dtype", [(1, 3, 1000, 128, True, torch.bfloat16),
                                                     (2, 2, 300, 64, False, torch.float32),
                                                     (1, 2, 513, 256, True, torch.float32)])
def test_noalloc_matches_oracle_and_attn_fwd_on_two_calls(B, H, N, d, causal, o_dtype):
    ea_build.build()
    (qn, kn, vn), (q, k, v) = device_qkv(B, H, N, d, seed=N + d)
    o_ref, lse_ref = ea.attn_fwd(q, k, v, causal=causal, o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    for call in range(2):
        o = torch.full(q.shape, float("nan"), dtype=o_dtype, device=q.device)
        lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=q.device)
        assert _call_noalloc(q, k, v, o, lse, causal) == ea.ATTN_OK, call
        torch.cuda.synchronize()
        assert ea.attn_noalloc_status() == ea.ATTN_OK, call
        assert_within(compare_full(o, lse, qn, kn, vn, 1.0 / math.sqrt(d), causal), ("oracle", call))
        diff = (o.float() - o_ref.float()).abs()
        assert diff.max().item() <= O_MAX_ABS and diff.mean().item() <= O_MEAN_ABS, call
        assert ((lse - lse_ref).abs() / lse_ref.abs()).max().item() <= LSE_REL, call


@pytest.mark.parametrize("B,H,N,d", [(2, 16, 8192, 128), (1, 32, 4096, 64), (2, 4, 2000, 256)])
def test_work_lists_do_not_change_results(B, H, N, d):
    """attn_fwd follows the host-built work lists (attn_fwd_schedule), attn_fwd_noalloc the
    round-robin order: every unit is computed the same way whichever CTA takes it, so O and LSE
    are bit-identical (causal, where the two orders differ most)."""
    ea_build.build()
    assert ea.attn_fwd_schedule(B, H, N, N, d, causal=True) is not None
    g = torch.Generator(device="cuda").manual_seed(N + d)
    q, k, v = (torch.randn(B, H, N, d, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3))
    o_ref, lse_ref = ea.attn_fwd(q, k, v, causal=True)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    assert _call_noalloc(q, k, v, o, lse, True) == ea.ATTN_OK
    torch.cuda.synchronize()
    assert ea.attn_noalloc_status() == ea.ATTN_OK and ea.attn_device_status() == ea.ATTN_OK
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_noalloc_status_reports_a_timeout_once():
    """A bounded wait that runs out, recorded in the static status word (the self-test kernel
    waits on a barrier that nothing arrives at, for 2 s), is reported by attn_noalloc_status,
    cleared by that read, and not seen by attn_device_status; the next call is still correct."""
    ea_build.build()
    assert ea.attn_noalloc_status() == ea.ATTN_OK
    ea.attn_noalloc_selftest_wait_timeout()
    assert ea.attn_noalloc_status() == ea.ATTN_ERR_TIMEOUT
    assert ea.attn_noalloc_status() == ea.ATTN_OK
    assert ea.attn_device_status() == ea.ATTN_OK
    (qn, kn, vn), (q, k, v) = device_qkv(1, 2, 300, 128, seed=4)
    o = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse = torch.empty((1, 2, 300), dtype=torch.float32, device=q.device)
    assert _call_noalloc(q, k, v, o, lse, True) == ea.ATTN_OK
    torch.cuda.synchronize()
    assert ea.attn_noalloc_status() == ea.ATTN_OK
    assert_within(compare_full(o, lse, qn, kn, vn, 1.0 / math.sqrt(128), True), "after timeout")


_CHILD = r"""
import json, math, sys
import torch
sys.path.insert(0, sys.argv[1])
import exact_attention_100_b200 as ea
from exact_attention_100_b200.inputs import normal_qkv
from oracle import attention_ref
import numpy as np
torch.cuda.set_device(0)
shapes = [(1, 2, 384, 64, True), (2, 1, 300, 128, False), (1, 1, 257, 256, True)]
bufs = []
for (B, H, N, d, causal) in shapes:
    qn, kn, vn = normal_qkv(B, H, N, d, seed=N)
    t = [torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (qn, kn, vn)]
    o = torch.empty(t[0].shape, dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    bufs.append(((qn, kn, vn), t, o, lse, causal))
torch.cuda.synchronize()
def run_all():
    for (_, (q, k, v), o, lse, causal) in bufs:
        ea.attn_fwd_noalloc(q, k, v, o, lse, causal=causal)
    torch.cuda.synchronize()
run_all()  # first calls: per-device set-up (every kernel module is loaded already: eager loading)
free0 = torch.cuda.mem_get_info()[0]
for _ in range(3):
    run_all()
free1 = torch.cuda.mem_get_info()[0]
status = ea.attn_noalloc_status()
errs = []
for ((qn, kn, vn), _, o, lse, causal) in bufs:
    d = qn.shape[-1]
    o_ref, lse_ref = attention_ref(qn, kn, vn, 1.0 / math.sqrt(d), causal)
    e = np.abs(o.cpu().numpy() - o_ref)
    errs.append([float(e.max()), float(e.mean()),
                 float((np.abs(lse.cpu().numpy() - lse_ref) / np.abs(lse_ref)).max())])
print(json.dumps({"free0": free0, "free1": free1, "status": status, "errs": errs}))
"""


def test_noalloc_in_a_fresh_process_allocates_nothing_per_call():
    """In a fresh process that never calls attn_fwd (so the library's own workspace is never
    created), with every kernel module loaded eagerly: after the first call of each shape, nine
    more calls over three head dims leave the device's free memory unchanged, the status word
    reads ATTN_OK, and every result meets the oracle's parity bars."""
    ea_build.build()
    env = dict(os.environ, CUDA_MODULE_LOADING="EAGER")
    r = subprocess.run([sys.executable, "-c", _CHILD, ROOT], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["status"] == ea.ATTN_OK
    assert res["free0"] == res["free1"], res
    for e in res["errs"]:
        assert e[0] <= O_MAX_ABS and e[1] <= O_MEAN_ABS and e[2] <= LSE_REL, e


def test_noalloc_rejects_bad_arguments_without_launching():
    ea_build.build()
    null = ctypes.c_void_p(0)
    p = ctypes.c_void_p(0x10000)
    f = ea.lib().attn_fwd_noalloc
    assert f(null, p, p, p, null, 1, 1, 128, 128, 0.1, 0, 0, 0, null) == ea.ATTN_ERR_INVALID_ARG
    assert f(p, p, p, p, null, 1, 1, 128, 96, 0.1, 0, 0, 0, null) == ea.ATTN_ERR_UNSUPPORTED
