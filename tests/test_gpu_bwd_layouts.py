"""The backward pass on strided tensors (attn_bwd_strided) and on packed batches of sequences of
different lengths (attn_bwd_varlen): against the float64 oracle with the derived elementwise
bound of test_gpu_bwd.py, and bit for bit against attn_bwd_qk on contiguous copies (the
arithmetic of a tile does not depend on where its rows are stored)."""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200.inputs import normal_dout, normal_qkv_lengths, normal_qkv_packed
from oracle import attention_ref, attention_bwd_chunked_ref, attention_bwd_ref, attention_varlen_bwd_ref

from test_gpu_bwd import _bounds

pytestmark = pytest.mark.gpu


def _check_grads(grads, refs, bounds):
    for name, g, r, b in zip(("dq", "dk", "dv"), grads, refs, bounds):
        g = np.asarray(g, dtype=np.float64)
        assert np.isfinite(g).all(), name
        tol = 2.0 * b + 1e-6 * (np.abs(r).max() if r.size else 0.0)
        err = np.abs(g - r)
        assert np.all(err[tol == 0] == 0), name
        worst = float(np.divide(err, tol, out=np.zeros_like(err), where=tol > 0).max()) if err.size else 0.0
        assert worst <= 1.0, (name, worst)


def _seq_major(t):
    """[B, H, N, d] device tensor -> the same values as a [B, H, N, d] view of [B, N, H, d] memory."""
    return t.transpose(1, 2).contiguous().transpose(1, 2)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,Nq,Nk,d", [(2, 2, 300, 300, 128), (1, 3, 129, 400, 64), (1, 2, 513, 130, 128)])
def test_strided_matches_contiguous_and_oracle(B, H, Nq, Nk, d, causal):
    q, k, v = normal_qkv_lengths(B, H, Nq, Nk, d, seed=1)
    do = normal_dout(B, H, Nq, d, seed=2)
    tq, tk, tv, tdo = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v, do))
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd_qk(tq, tk, tv, scale=scale, causal=causal)
    ref = ea.attn_bwd_qk(tq, tk, tv, o, lse, tdo, scale=scale, causal=causal, g_dtype=torch.float32)
    sq, sk, sv, so, sdo = (_seq_major(t) for t in (tq, tk, tv, o, tdo))
    got = ea.attn_bwd_strided(sq, sk, sv, so, lse, sdo, scale=scale, causal=causal, g_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    assert got[0].stride() == sq.stride()  # gradients come back in the inputs' memory order
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    o_ref, _ = attention_ref(q, k, v, scale, causal)
    _check_grads([g.cpu().numpy() for g in got], attention_bwd_ref(q, k, v, do, scale, causal),
                 _bounds(q, k, v, do, o_ref, scale, causal))


def test_strided_gradients_into_a_fused_buffer():
    """dQ, dK, dV written as slices of one [B, N, 3, H, d] buffer; nothing else is touched."""
    B, H, N, d = 1, 4, 257, 64
    q, k, v = normal_qkv_lengths(B, H, N, N, d, seed=3)
    do = normal_dout(B, H, N, d, seed=4)
    tq, tk, tv, tdo = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v, do))
    o, lse = ea.attn_fwd(tq, tk, tv, causal=True)
    ref = ea.attn_bwd(tq, tk, tv, o, lse, tdo, causal=True)
    buf = torch.full((B, N, 4, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    dq, dk, dv = (buf[:, :, i].transpose(1, 2) for i in range(3))
    ea.attn_bwd_strided(tq, tk, tv, o, lse, tdo, dq=dq, dk=dk, dv=dv, causal=True)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    assert torch.isnan(buf[:, :, 3]).all()
    for a, b in zip((dq, dk, dv), ref):
        assert torch.equal(a, b)


def _packed_run(lq, lk, H, d, causal, seed, layout="plain", ds=False):
    q, k, v, cq, ck = normal_qkv_packed(lq, lk, H, d, seed=seed)
    do = np.random.default_rng(seed + 100).standard_normal(q.shape).astype(np.float32)
    from exact_attention_100_b200.inputs import round_to_bf16
    do = round_to_bf16(do)
    if layout == "fused":
        qkv = torch.from_numpy(np.stack([q, k, v], axis=1)).to(torch.bfloat16).cuda()
        tq, tk, tv = qkv[:, 0], qkv[:, 1], qkv[:, 2]
    else:
        tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    tdo = torch.from_numpy(do).to(torch.bfloat16).cuda()
    tcq, tck = torch.from_numpy(cq).cuda(), torch.from_numpy(ck).cuda()
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd_varlen(tq, tk, tv, tcq, tck, max(lq), scale=scale, causal=causal)
    bwd = ea.attn_bwd_varlen_ds if ds else ea.attn_bwd_varlen
    grads = bwd(tq, tk, tv, o, lse, tdo, tcq, tck, max(lq), max(lk), scale=scale, causal=causal, g_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    if ds:
        # dK and dV come from the same dK/dV arithmetic as attn_bwd_varlen: the same bits
        ref = ea.attn_bwd_varlen(tq, tk, tv, o, lse, tdo, tcq, tck, max(lq), max(lk), scale=scale, causal=causal,
                                 g_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(grads[1], ref[1]) and torch.equal(grads[2], ref[2])
    return (q, k, v, do, cq, ck, scale), (tq, tk, tv, tdo, o, lse), [g.cpu().numpy() for g in grads]


def _check_packed(inputs, grads, causal):
    q, k, v, do, cq, ck, scale = inputs
    refs = attention_varlen_bwd_ref(q, k, v, do, cq, ck, scale, causal)
    t = lambda x: x.transpose(1, 0, 2)[None]  # [rows, H, d] -> [1, H, rows, d]
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        gs = [t(grads[0][q0:q1]), t(grads[1][k0:k1]), t(grads[2][k0:k1])]
        rs = [t(refs[0][q0:q1]), t(refs[1][k0:k1]), t(refs[2][k0:k1])]
        if q1 == q0 or k1 == k0:
            for g in gs:
                assert np.all(g == 0)  # no queries or no keys: zero gradients
            continue
        qs, ks, vs, dos = t(q[q0:q1]), t(k[k0:k1]), t(v[k0:k1]), t(do[q0:q1])
        o_ref, _ = attention_ref(qs, ks, vs, scale, causal)
        _check_grads(gs, rs, _bounds(qs, ks, vs, dos, o_ref, scale, causal))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_packed_matches_oracle(d, causal):
    lq = [300, 1, 129, 128, 513, 127]
    inputs, _, grads = _packed_run(lq, lq, 2, d, causal, seed=5)
    _check_packed(inputs, grads, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_packed_lengths_differ_per_sequence(causal):
    """Per-sequence Nq != Nk, an empty query sequence, an empty key sequence, rows that see no key
    and keys that no query sees."""
    lq = [200, 0, 64, 700, 130, 5]
    lk = [90, 17, 0, 260, 600, 1]
    inputs, _, grads = _packed_run(lq, lk, 2, 128, causal, seed=6)
    _check_packed(inputs, grads, causal)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lk,layout", [([257, 40, 600], "fused"), ([300, 40, 129], "plain")])
def test_packed_is_per_sequence_attn_bwd_qk(lk, layout, causal):
    """Each sequence's gradients are the bits attn_bwd_qk gives on that sequence alone (Q, K, V
    as slices of one fused buffer when the lengths agree)."""
    lq = [257, 40, 600]
    (q, k, v, do, cq, ck, scale), (tq, tk, tv, tdo, o, lse), grads = _packed_run(lq, lk, 2, 64, causal, seed=7,
                                                                                 layout=layout)
    for b in range(3):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        t = lambda x: x.transpose(0, 1).unsqueeze(0).contiguous()
        ref = ea.attn_bwd_qk(t(tq[q0:q1]), t(tk[k0:k1]), t(tv[k0:k1]), t(o[q0:q1]), lse[:, q0:q1].unsqueeze(0).contiguous(),
                             t(tdo[q0:q1]), scale=scale, causal=causal, g_dtype=torch.float32)
        torch.cuda.synchronize()
        back = lambda g: g[0].transpose(0, 1).cpu().numpy()
        assert np.array_equal(grads[0][q0:q1], back(ref[0]))
        assert np.array_equal(grads[1][k0:k1], back(ref[1]))
        assert np.array_equal(grads[2][k0:k1], back(ref[2]))


@pytest.mark.parametrize("causal", [True, False])
def test_packed_bench_batch_two_heads(causal):
    """The bench's packed workload (8 sequences of 391..3369 tokens, 16384 in all, H=16 d=128,
    seed 11): every sequence of heads 0 and 15 against the float64 oracle under the derived
    bound (oracle and bound taken 1024 query rows at a time)."""
    from bench import VARLEN_WORKLOAD, varlen_lengths
    w = VARLEN_WORKLOAD
    lens = varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
    assert sum(lens) == w["total"] and len(lens) == 8
    (q, k, v, do, cq, ck, scale), _, grads = _packed_run(lens, lens, w["H"], w["d"], causal, seed=w["seed"])
    for h in (0, w["H"] - 1):
        for b in range(len(lens)):
            q0, q1 = int(cq[b]), int(cq[b + 1])
            t = lambda x: x[q0:q1, h][None, None]  # [1, 1, rows, d]
            qs, ks, vs, dos = t(q), t(k), t(v), t(do)
            refs = attention_bwd_chunked_ref(qs, ks, vs, dos, scale, causal)
            o_ref, _ = attention_ref(qs, ks, vs, scale, causal)
            _check_grads([t(g) for g in grads], refs, _bounds(qs, ks, vs, dos, o_ref, scale, causal))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_packed_ds_matches_oracle(d, causal):
    """attn_bwd_varlen_ds (dS kept in the workspace): the same bound per sequence, dK and dV the
    bits of attn_bwd_varlen."""
    lq = [300, 1, 129, 128, 513, 127]
    inputs, _, grads = _packed_run(lq, lq, 2, d, causal, seed=15, ds=True)
    _check_packed(inputs, grads, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_packed_ds_lengths_differ_per_sequence(causal):
    lq = [200, 0, 64, 700, 130, 5]
    lk = [90, 17, 0, 260, 600, 1]
    inputs, _, grads = _packed_run(lq, lk, 2, 128, causal, seed=16, ds=True)
    _check_packed(inputs, grads, causal)


def test_packed_ds_bench_batch_two_heads():
    """The bench's packed workload through attn_bwd_varlen_ds, causal: every sequence of heads 0
    and 15 against the float64 oracle under the derived bound."""
    from bench import VARLEN_WORKLOAD, varlen_lengths
    w = VARLEN_WORKLOAD
    lens = varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
    (q, k, v, do, cq, ck, scale), _, grads = _packed_run(lens, lens, w["H"], w["d"], True, seed=w["seed"], ds=True)
    for h in (0, w["H"] - 1):
        for b in range(len(lens)):
            q0, q1 = int(cq[b]), int(cq[b + 1])
            t = lambda x: x[q0:q1, h][None, None]
            qs, ks, vs, dos = t(q), t(k), t(v), t(do)
            refs = attention_bwd_chunked_ref(qs, ks, vs, dos, scale, True)
            o_ref, _ = attention_ref(qs, ks, vs, scale, True)
            _check_grads([t(g) for g in grads], refs, _bounds(qs, ks, vs, dos, o_ref, scale, True))


@pytest.mark.parametrize("ds", [False, True])
def test_packed_bad_offsets_are_reported(ds):
    lq = [300, 200, 250]
    q, k, v, cq, ck = normal_qkv_packed(lq, lq, 2, 64, seed=8)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    tcq, tck = torch.from_numpy(cq).cuda(), torch.from_numpy(ck).cuda()
    o, lse = ea.attn_fwd_varlen(tq, tk, tv, tcq, tck, 300, causal=True)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    bad = tcq.clone()
    bad[2] = 100  # sequence 1 decreasing, sequence 2 longer than max_seqlen_q
    dq = torch.full(tq.shape, float("nan"), dtype=torch.float32, device="cuda")
    bwd = ea.attn_bwd_varlen_ds if ds else ea.attn_bwd_varlen
    bwd(tq, tk, tv, o, lse, torch.ones_like(tq), bad, tck, 300, 300, dq=dq, causal=True)
    assert ea.attn_device_status() == ea.ATTN_ERR_INVALID_ARG
    assert not torch.isnan(dq[:300]).any() and torch.isnan(dq[300:]).all()
