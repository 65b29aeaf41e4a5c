"""Seeded random shapes against the float64 oracle.

The other parity tests pick their shapes by hand (tile edges, one row, empty sequences, the
timed sizes); here a fixed seed draws further ones -- lengths anywhere in 1..900, query and key
lengths unrelated, head dims, causal or not, bf16 or float32 outputs -- so that a case nobody
thought of still meets the same bars: O within 1e-2 (max) and 1e-3 (mean) of the oracle, LSE
within 1e-3 relative, rows without a visible key exactly O = 0 and LSE = -inf; gradients within
the elementwise bound derived for the backward, and the dS-keeping backward's dK and dV the
same bits as the recomputing one's; the E4M3 forward on the pre-kernel's codes within its own
bars against the dequantised inputs; packed backwards whose key and query lengths differ."""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build
from exact_attention_100_b200.inputs import hadamard_signs, normal_dout, normal_qkv_lengths, normal_qkv_packed
from oracle import attention_ref, attention_varlen_ref, dequant_ref

from gpu_util import LSE_REL, O_MAX_ABS, O_MEAN_ABS
from test_gpu_bwd import _check
from test_gpu_bwd_layouts import _check_packed

pytestmark = pytest.mark.gpu

_RNG = np.random.default_rng(2026)
# causal and the output dtype alternate with the case index; the rest is drawn
FWD_CASES = [(int(_RNG.integers(1, 3)), int(_RNG.integers(1, 4)), int(_RNG.integers(1, 901)), int(_RNG.integers(1, 901)),
              int(_RNG.choice([64, 128, 256])), i % 2 == 1, i % 4 < 2) for i in range(16)]
BWD_CASES = [(int(_RNG.integers(1, 3)), int(_RNG.integers(1, 3)), int(_RNG.integers(1, 801)),
              int(_RNG.choice([64, 128])), i % 2 == 1) for i in range(8)]
VARLEN_CASES = [([int(x) for x in _RNG.integers(0, 600, size=int(_RNG.integers(1, 7)))],
                 int(_RNG.choice([64, 128, 256])), i % 2 == 1) for i in range(4)]
FP8_CASES = [(int(_RNG.integers(1, 901)), int(_RNG.integers(1, 901)), int(_RNG.choice([64, 128, 256])), i % 2 == 1)
             for i in range(6)]
VARLEN_BWD_CASES = [([int(x) for x in _RNG.integers(0, 500, size=int(_RNG.integers(1, 6)))],
                     [int(x) for x in _RNG.integers(0, 500, size=1)], int(_RNG.choice([64, 128])), i % 2 == 1)
                    for i in range(4)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ea_build.build()
    ea.lib()


def _fwd_check(o, lse, o_ref, lse_ref):
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty)
    assert np.all(o[empty] == 0.0)
    err = np.abs(o - o_ref)[~empty]
    if err.size:
        assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, (err.max(), err.mean())
        rel = np.abs(lse[~empty] - lse_ref[~empty]) / np.abs(lse_ref[~empty])
        assert rel.max() <= LSE_REL, rel.max()


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,f32", FWD_CASES)
def test_forward_random_shapes(B, H, Nq, Nk, d, causal, f32):
    q, k, v = normal_qkv_lengths(B, H, Nq, Nk, d, seed=Nq * 7 + Nk)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd_qk(tq, tk, tv, scale=scale, causal=causal, o_dtype=torch.float32 if f32 else torch.bfloat16)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    o_ref, lse_ref = attention_ref(q, k, v, scale, causal)
    _fwd_check(o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), o_ref, lse_ref)


@pytest.mark.parametrize("B,H,N,d,causal", BWD_CASES)
def test_backward_random_shapes(B, H, N, d, causal):
    q, k, v = normal_qkv_lengths(B, H, N, N, d, seed=N + d)
    do = normal_dout(B, H, N, d, seed=N + 3)
    tq, tk, tv, tdo = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v, do))
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd(tq, tk, tv, scale=scale, causal=causal)
    g = ea.attn_bwd(tq, tk, tv, o, lse, tdo, scale=scale, causal=causal, g_dtype=torch.float32)
    g_ds = ea.attn_bwd_ds(tq, tk, tv, o, lse, tdo, scale=scale, causal=causal, g_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    assert torch.equal(g[1], g_ds[1]) and torch.equal(g[2], g_ds[2])
    _check((q, k, v, do, scale), g, causal)
    _check((q, k, v, do, scale), g_ds, causal)


@pytest.mark.parametrize("lens,d,causal", VARLEN_CASES)
def test_packed_forward_random_lengths(lens, d, causal):
    H = 2
    q, k, v, cq, ck = normal_qkv_packed(lens, lens, H, d, seed=sum(lens) + d)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    tcq, tck = torch.from_numpy(cq).cuda(), torch.from_numpy(ck).cuda()
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd_varlen(tq, tk, tv, tcq, tck, max(max(lens), 1), scale=scale, causal=causal,
                                o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    o_ref, lse_ref = attention_varlen_ref(q, k, v, cq, ck, scale, causal)
    # O is [total, H, d] and LSE [H, total]: compare O as [H, total, d]
    _fwd_check(o.permute(1, 0, 2).cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
               np.transpose(o_ref, (1, 0, 2)), lse_ref)


@pytest.mark.parametrize("nq,nk,d,causal", FP8_CASES)
def test_fp8_forward_random_shapes(nq, nk, d, causal):
    """attn_fwd_fp8_qk on the pre-kernel's codes: the E4M3 bars against the oracle on the
    dequantised inputs (RMSE <= 1e-2, |error| <= (2^-4 + 1e-2) max|v|, LSE relative <= 1e-3)."""
    q, k, v = normal_qkv_lengths(1, 2, nq, nk, d, seed=nq * 3 + nk)
    dev = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda()
    signs = torch.from_numpy(hadamard_signs(d)).cuda()
    q8, qs = ea.attn_hadamard_quant(dev(q), signs)
    k8, ks = ea.attn_hadamard_quant(dev(k), signs)
    v8, vs = ea.attn_hadamard_quant(dev(v), None)
    o, lse = ea.attn_fwd_fp8_qk(q8, k8, v8, qs, ks, vs, causal=causal, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    qd, kd, vd = (dequant_ref(a.cpu().numpy(), s_.cpu().numpy()) for a, s_ in ((q8, qs), (k8, ks), (v8, vs)))
    o_ref, lse_ref = attention_ref(qd, kd, vd, 1 / math.sqrt(d), causal)
    og, lg = o.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lg), empty) and np.all(og[empty] == 0.0)
    err = (og - o_ref)[~empty]
    if err.size:
        assert float(np.sqrt(np.mean(err ** 2))) <= 1e-2
        assert np.abs(err).max() <= (2.0 ** -4 + 1e-2) * np.abs(vd).max()
        assert (np.abs(lg[~empty] - lse_ref[~empty]) / np.abs(lse_ref[~empty])).max() <= 1e-3


@pytest.mark.parametrize("lq,extra,d,causal", VARLEN_BWD_CASES)
def test_packed_backward_random_lengths(lq, extra, d, causal):
    """attn_bwd_varlen_ds on a packed batch whose key lengths differ from the query lengths
    (each sequence's keys are its query count plus or minus a drawn offset, empty ones too),
    per sequence against the oracle; dK and dV the bits of attn_bwd_varlen."""
    lk = [max(0, n + (extra[0] % 97) - 48) for n in lq]
    H = 2
    q, k, v, cq, ck = normal_qkv_packed(lq, lk, H, d, seed=sum(lq) + sum(lk) + d)
    do = normal_qkv_packed(lq, lq, H, d, seed=sum(lq) + 5)[0]
    tq, tk, tv, tdo = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v, do))
    tcq, tck = torch.from_numpy(cq).cuda(), torch.from_numpy(ck).cuda()
    scale = 1.0 / math.sqrt(d)
    mq, mk = max(max(lq), 1), max(max(lk), 1)
    o, lse = ea.attn_fwd_varlen(tq, tk, tv, tcq, tck, mq, scale=scale, causal=causal)
    g = ea.attn_bwd_varlen_ds(tq, tk, tv, o, lse, tdo, tcq, tck, mq, mk, scale=scale, causal=causal,
                              g_dtype=torch.float32)
    ref = ea.attn_bwd_varlen(tq, tk, tv, o, lse, tdo, tcq, tck, mq, mk, scale=scale, causal=causal,
                             g_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    assert torch.equal(g[1], ref[1]) and torch.equal(g[2], ref[2])
    _check_packed((q, k, v, do, cq, ck, scale), [x.cpu().numpy() for x in g], causal)

