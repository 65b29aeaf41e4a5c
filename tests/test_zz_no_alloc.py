"""The allocation-free entry point, attn_fwd_noalloc, against attn_fwd (GPU).

attn_fwd_noalloc is for callers that cannot let the library call cudaMalloc (runtimes that
own all device memory through their own pool, hosts with a fixed memory budget, loops that
must never reach an allocation that may synchronise the device): its scratch is a static
device array of the library.  Its results must match attn_fwd's within the parity tolerances
of the other GPU tests, on two calls in a row (the second call finds the array holding the
first call's contents).  This file is collected last on purpose.
"""

import ctypes
import math

import pytest

torch = pytest.importorskip("torch")

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build
from gpu_util import LSE_REL, O_MAX_ABS, O_MEAN_ABS, device_qkv

pytestmark = pytest.mark.gpu


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
def test_noalloc_matches_attn_fwd_on_two_calls(B, H, N, d, causal, o_dtype):
    ea_build.build()
    _, (q, k, v) = device_qkv(B, H, N, d, seed=N + d)
    o_ref, lse_ref = ea.attn_fwd(q, k, v, causal=causal, o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    for call in range(2):
        o = torch.full(q.shape, float("nan"), dtype=o_dtype, device=q.device)
        lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=q.device)
        assert _call_noalloc(q, k, v, o, lse, causal) == ea.ATTN_OK, call
        torch.cuda.synchronize()
        diff = (o.float() - o_ref.float()).abs()
        assert diff.max().item() <= O_MAX_ABS and diff.mean().item() <= O_MEAN_ABS, call
        assert ((lse - lse_ref).abs() / lse_ref.abs()).max().item() <= LSE_REL, call


def test_noalloc_rejects_bad_arguments_without_launching():
    ea_build.build()
    null = ctypes.c_void_p(0)
    p = ctypes.c_void_p(0x10000)
    f = ea.lib().attn_fwd_noalloc
    assert f(null, p, p, p, null, 1, 1, 128, 128, 0.1, 0, 0, 0, null) == ea.ATTN_ERR_INVALID_ARG
    assert f(p, p, p, p, null, 1, 1, 128, 96, 0.1, 0, 0, 0, null) == ea.ATTN_ERR_UNSUPPORTED
