"""attn_fwd_varlen: packed batches of sequences of different lengths against the float64
oracle (``attention_varlen_ref``), bit for bit against attn_fwd when every length is equal,
and the device-side check of the sequence offsets."""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200.inputs import normal_qkv_packed, uniform_lengths
from oracle import attention_varlen_ref

from gpu_util import LSE_REL, O_MAX_ABS, O_MEAN_ABS

pytestmark = pytest.mark.gpu


def _dev(*arrays):
    out = []
    for a in arrays:
        t = torch.from_numpy(np.ascontiguousarray(a))
        out.append((t.to(torch.bfloat16) if t.dtype == torch.float32 else t).cuda())
    return out


def _check(o, lse, q, k, v, cu_q, cu_k, scale, causal):
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    o_ref, lse_ref = attention_varlen_ref(q, k, v, cu_q, cu_k, scale, causal)
    empty = np.isneginf(lse_ref)  # [H, total_q]: rows with no visible key
    assert np.array_equal(np.isneginf(lse), empty)
    assert np.all(o.transpose(1, 0, 2)[empty] == 0.0)
    err = np.abs(o - o_ref).transpose(1, 0, 2)[~empty]
    if err.size:
        assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, (err.max(), err.mean())
        rel = np.abs(lse[~empty] - lse_ref[~empty]) / np.abs(lse_ref[~empty])
        assert rel.max() <= LSE_REL, rel.max()


def _run(lq, lk, H, d, causal, seed=0, o_dtype=torch.float32):
    q, k, v, cu_q, cu_k = normal_qkv_packed(lq, lk, H, d, seed=seed)
    tq, tk, tv, tcq, tck = _dev(q, k, v, cu_q, cu_k)
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd_varlen(tq, tk, tv, tcq, tck, max(lq), scale=scale, causal=causal, o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    _check(o, lse, q, k, v, cu_q, cu_k, scale, causal)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_mixed_lengths_match_oracle(d, causal):
    """Lengths across tile boundaries: 1, 127, 128, 129, 300, 513 queries; keys equal."""
    lq = [300, 1, 129, 128, 513, 127]
    _run(lq, lq, 2, d, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_query_and_key_lengths_differ_per_sequence(causal):
    """Per-sequence Nq != Nk with bottom-right alignment, an empty query sequence, an empty
    key sequence (its rows get O = 0, LSE = -inf) and rows that see no key."""
    lq = [200, 0, 64, 700, 130, 5]
    lk = [90, 17, 0, 260, 600, 1]
    _run(lq, lk, 3, 128, causal, seed=1)


@pytest.mark.parametrize("causal", [False, True])
def test_random_length_mix(causal):
    lq = [int(x) for x in uniform_lengths(12, 1, 1100, seed=3)]
    _run(lq, lq, 2, 128, causal, seed=2)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_are_attn_fwd(causal):
    """Every sequence of length N: same bits as the fixed-length kernel on the unpacked batch
    (rows of the next sequence read past a sequence's end get exactly zero weight)."""
    B, H, N, d = 3, 2, 333, 128
    q, k, v, cu_q, cu_k = normal_qkv_packed([N] * B, [N] * B, H, d, seed=4)
    tq, tk, tv, tcq, tck = _dev(q, k, v, cu_q, cu_k)
    o, lse = ea.attn_fwd_varlen(tq, tk, tv, tcq, tck, N, causal=causal)
    unpack = lambda t: t.view(B, N, H, d).transpose(1, 2).contiguous()
    of, lf = ea.attn_fwd(unpack(tq), unpack(tk), unpack(tv), causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o, of.transpose(1, 2).reshape(B * N, H, d))
    assert torch.equal(lse, lf.transpose(0, 1).reshape(H, B * N))


def test_fused_qkv_packed_layout():
    """q, k, v as slices of one [total, 3, H, d] buffer (row stride 3 H d)."""
    lq = [257, 40, 600]
    H, d = 4, 64
    q, k, v, cu_q, cu_k = normal_qkv_packed(lq, lq, H, d, seed=5)
    qkv = torch.from_numpy(np.stack([q, k, v], axis=1)).to(torch.bfloat16).cuda()
    tcq, tck = _dev(cu_q, cu_k)
    o, lse = ea.attn_fwd_varlen(qkv[:, 0], qkv[:, 1], qkv[:, 2], tcq, tck, max(lq), causal=True,
                                o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    _check(o, lse, q, k, v, cu_q, cu_k, 1.0 / math.sqrt(d), True)


def test_bad_offsets_are_reported_and_skipped():
    """A decreasing offset pair and a sequence longer than max_seqlen_q are found on the device:
    those sequences are skipped, attn_device_status reports ATTN_ERR_INVALID_ARG, and the
    other sequences are still computed."""
    lq = [300, 200, 250]
    q, k, v, cu_q, cu_k = normal_qkv_packed(lq, lq, 2, 128, seed=6)
    tq, tk, tv, tcq, tck = _dev(q, k, v, cu_q, cu_k)
    bad_q = tcq.clone()
    bad_q[2] = 100  # sequence 1 becomes [300, 100): decreasing; sequence 2 [100, 750) too long
    o = torch.full((q.shape[0], 2, 128), float("nan"), dtype=torch.float32, device="cuda")
    _, lse = ea.attn_fwd_varlen(tq, tk, tv, bad_q, tck, 300, o=o, causal=True)
    assert ea.attn_device_status() == ea.ATTN_ERR_INVALID_ARG
    assert ea.attn_device_status() == ea.ATTN_OK  # the report is cleared
    # sequence 0 is intact; rows of the skipped sequences are untouched
    o_ref, lse_ref = attention_varlen_ref(q, k, v, cu_q, cu_k, 1.0 / math.sqrt(128), True)
    assert np.abs(o[:300].cpu().numpy() - o_ref[:300]).max() <= O_MAX_ABS
    assert torch.isnan(o[300:]).all()
    # max_seqlen_q smaller than a sequence: that sequence is skipped and reported
    o.fill_(float("nan"))
    ea.attn_fwd_varlen(tq, tk, tv, tcq, tck, 250, o=o, causal=False)
    assert ea.attn_device_status() == ea.ATTN_ERR_INVALID_ARG
    assert torch.isnan(o[:300]).all() and not torch.isnan(o[300:]).any()


@pytest.mark.parametrize("causal", [False, True])
def test_more_sequences_than_the_schedule_holds(causal):
    """1100 short sequences: more than the in-kernel schedule's 1024, so the launch deals out
    units in the plain round order (empty ones skipped) -- same results."""
    lq = [int(x) for x in uniform_lengths(1100, 1, 24, seed=9)]
    _run(lq, lq, 1, 64, causal, seed=10)


def test_schedule_covers_sequences_of_one_length_and_empty_ones():
    """Sorting by tile pairs with many ties and zero-length sequences in between."""
    lq = [256, 0, 256, 512, 0, 1, 256, 257, 0, 512]
    _run(lq, lq, 2, 128, True, seed=11)


@pytest.mark.parametrize("causal", [True, False])
def test_bench_packed_batch_all_heads(causal):
    """The packed batch the bench times: 8 sequences of 391..3369 tokens (16384 in all), H=16
    d=128, seed 11, bf16 O; every row of every head against the float64 oracle."""
    from bench import VARLEN_WORKLOAD, varlen_lengths
    w = VARLEN_WORKLOAD
    lens = varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
    assert sum(lens) == w["total"] and len(lens) == 8
    _run(lens, lens, w["H"], w["d"], causal, seed=w["seed"], o_dtype=torch.bfloat16)
