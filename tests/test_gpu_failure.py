"""Failure detection on the GPU without a fault: the library's bounded mbarrier wait, made to
run out by a barrier that nothing arrives at, records a timeout that attn_device_status
reports; the kernel returns and the context keeps working."""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from oracle import attention_ref

from gpu_util import device_qkv

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_and_the_context_survives():
    assert ea.attn_device_status() == ea.ATTN_OK
    ea.attn_selftest_wait_timeout()
    assert ea.attn_device_status() == ea.ATTN_ERR_TIMEOUT  # synchronises: the kernel returned
    assert ea.attn_device_status() == ea.ATTN_OK  # the report is cleared
    (q, k, v), (tq, tk, tv) = device_qkv(1, 2, 300, 128, seed=31)
    o, lse = ea.attn_fwd(tq, tk, tv, causal=True, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    o_ref, _ = attention_ref(q, k, v, 1.0 / math.sqrt(128), True)
    assert np.abs(o.cpu().numpy() - o_ref).max() <= 1e-2
