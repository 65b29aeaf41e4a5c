"""attn_fwd_qk: key/value length Nk different from the query length Nq, against the float64
oracle (which takes the bottom-right causal alignment, j <= i + Nk - Nq, and gives O = 0,
LSE = -inf to a row with no visible key)."""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200.inputs import normal_qkv_lengths
from oracle import attention_ref

from gpu_util import LSE_REL, O_MAX_ABS, O_MEAN_ABS

pytestmark = pytest.mark.gpu


def _run(B, H, Nq, Nk, d, causal, o_dtype=torch.float32, seed=0):
    q, k, v = normal_qkv_lengths(B, H, Nq, Nk, d, seed=seed)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd_qk(tq, tk, tv, scale=scale, causal=causal, o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    return (q, k, v, scale), (o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,Nq,Nk,d", [
    (1, 2, 128, 300, 128), (1, 2, 300, 128, 128), (1, 1, 1, 513, 64), (1, 1, 513, 1, 64),
    (2, 2, 200, 700, 256), (1, 2, 384, 256, 128), (1, 1, 129, 1000, 128), (1, 3, 1000, 129, 64),
    (1, 1, 640, 130, 128), (2, 1, 257, 257, 128),
])
def test_fwd_qk_matches_oracle(B, H, Nq, Nk, d, causal):
    (q, k, v, scale), (o, lse) = _run(B, H, Nq, Nk, d, causal)
    o_ref, lse_ref = attention_ref(q, k, v, scale, causal)
    empty = np.isneginf(lse_ref)  # rows that see no key
    assert np.array_equal(np.isneginf(lse), empty)
    assert np.all(o[empty] == 0.0)
    err = np.abs(o - o_ref)[~empty]
    if err.size:
        assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, (err.max(), err.mean())
        rel = np.abs(lse[~empty] - lse_ref[~empty]) / np.abs(lse_ref[~empty])
        assert rel.max() <= LSE_REL, rel.max()


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_qk_equal_lengths_is_attn_fwd(causal):
    q, k, v = normal_qkv_lengths(1, 2, 500, 500, 128, seed=3)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    a = ea.attn_fwd(tq, tk, tv, causal=causal)
    b = ea.attn_fwd_qk(tq, tk, tv, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fwd_qk_decode_shape():
    """One query row against a long cache (decode): causal and not coincide."""
    (q, k, v, scale), (o1, l1) = _run(2, 4, 1, 4096, 128, True, seed=5)
    (_, _, _, _), (o0, l0) = _run(2, 4, 1, 4096, 128, False, seed=5)
    assert np.array_equal(o1, o0) and np.array_equal(l1, l0)
    o_ref, lse_ref = attention_ref(q, k, v, scale, False)
    assert np.abs(o1 - o_ref).max() <= O_MAX_ABS
