"""attn_fwd_strided: Q, K, V read and O written through caller-given strides (sequence-major
[B, N, H, d], a fused [B, N, 3, H, d] projection, padded rows), against the float64 oracle and
bit for bit against attn_fwd_qk on contiguous copies (the arithmetic does not depend on the
addressing)."""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200.inputs import normal_qkv_lengths
from oracle import attention_ref

from gpu_util import LSE_REL, O_MAX_ABS, O_MEAN_ABS

pytestmark = pytest.mark.gpu


def _check_oracle(o, lse, q, k, v, scale, causal):
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    o_ref, lse_ref = attention_ref(q, k, v, scale, causal)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty)
    assert np.all(o[empty] == 0.0)
    err = np.abs(o - o_ref)[~empty]
    if err.size:
        assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, (err.max(), err.mean())
        rel = np.abs(lse[~empty] - lse_ref[~empty]) / np.abs(lse_ref[~empty])
        assert rel.max() <= LSE_REL, rel.max()


def _seq_major(a):
    """[B, H, N, d] host array -> [B, H, N, d] view of a [B, N, H, d] contiguous device tensor."""
    t = torch.from_numpy(np.ascontiguousarray(a.transpose(0, 2, 1, 3))).to(torch.bfloat16).cuda()
    return t.transpose(1, 2)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,Nq,Nk,d", [
    (2, 3, 300, 300, 128), (1, 2, 129, 700, 64), (2, 2, 200, 200, 256), (1, 4, 513, 130, 128),
    (1, 1, 1, 300, 128),
])
def test_sequence_major_matches_oracle(B, H, Nq, Nk, d, causal):
    q, k, v = normal_qkv_lengths(B, H, Nq, Nk, d, seed=1)
    tq, tk, tv = _seq_major(q), _seq_major(k), _seq_major(v)
    assert not tq.is_contiguous() or H == 1
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd_strided(tq, tk, tv, scale=scale, causal=causal, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    assert o.stride() == tq.stride()  # O comes back sequence-major too
    _check_oracle(o, lse, q, k, v, scale, causal)
    # same bits as the contiguous entry point
    ref = ea.attn_fwd_qk(tq.contiguous(), tk.contiguous(), tv.contiguous(), scale=scale, causal=causal,
                         o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_fused_qkv_projection_layout(d, causal):
    """q, k, v as slices of one [B, N, 3, H, d] buffer; bf16 O into a slice of a wider buffer
    whose other columns must stay untouched."""
    B, H, N = 2, 4, 333
    q, k, v = normal_qkv_lengths(B, H, N, N, d, seed=2)
    host = np.stack([a.transpose(0, 2, 1, 3) for a in (q, k, v)], axis=2)  # [B, N, 3, H, d]
    qkv = torch.from_numpy(np.ascontiguousarray(host)).to(torch.bfloat16).cuda()
    tq, tk, tv = (qkv[:, :, i].transpose(1, 2) for i in range(3))
    wide = torch.full((B, N, H, 2 * d), float("nan"), dtype=torch.bfloat16, device="cuda")
    o = wide[..., :d].transpose(1, 2)
    _, lse = ea.attn_fwd_strided(tq, tk, tv, o=o, causal=causal)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    assert torch.isnan(wide[..., d:]).all()
    ref = ea.attn_fwd(tq.contiguous(), tk.contiguous(), tv.contiguous(), causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1])
    _check_oracle(o, lse, q, k, v, 1.0 / math.sqrt(d), causal)


def test_padded_rows_and_mixed_layouts():
    """Each tensor with its own layout: q head-major with padded rows, k sequence-major, v
    contiguous, O head-major with a padded batch stride."""
    B, H, Nq, Nk, d = 2, 2, 260, 390, 128
    q, k, v = normal_qkv_lengths(B, H, Nq, Nk, d, seed=4)
    qpad = torch.zeros((B, H, Nq, d + 64), dtype=torch.bfloat16, device="cuda")
    qpad[..., :d] = torch.from_numpy(q).to(torch.bfloat16)
    tq = qpad[..., :d]
    tk = _seq_major(k)
    tv = torch.from_numpy(v).to(torch.bfloat16).cuda()
    obuf = torch.full((B, H * Nq * d + 256), float("nan"), dtype=torch.float32, device="cuda")
    o = obuf[:, : H * Nq * d].view(B, H, Nq, d)
    _, lse = ea.attn_fwd_strided(tq, tk, tv, o=o, causal=True)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    assert torch.isnan(obuf[:, H * Nq * d:]).all()
    ref = ea.attn_fwd_qk(tq.contiguous(), tk.contiguous(), tv, causal=True, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1])
    _check_oracle(o, lse, q, k, v, 1.0 / math.sqrt(d), True)


def test_contiguous_strides_are_attn_fwd():
    q, k, v = normal_qkv_lengths(1, 2, 400, 400, 128, seed=6)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    a = ea.attn_fwd(tq, tk, tv, causal=True)
    b = ea.attn_fwd_strided(tq, tk, tv, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_rejects_unaligned_row_stride():
    """A row stride of 100 elements (200 bytes) is not a multiple of 16 bytes."""
    x = torch.zeros((1, 1, 256, 100), dtype=torch.bfloat16, device="cuda")[..., :64]
    with pytest.raises(ea.AttnError):
        ea.attn_fwd_strided(x, x, x)
