"""Parity of the backward pass (attn_bwd, through the C ABI) with the float64 oracle.

Tolerance, derived from the arithmetic rather than fitted (u = 2^-9, the bf16 unit roundoff;
all products elementwise in absolute value, everything from the oracle in float64):

* P is recomputed in float32 from the forward's LSE (relative error < 1e-4: scores summed in
  float32, ex2.approx or a cubic with relative error < 7.5e-5) and rounded to bf16 (u):
                                                          dP_err  <= (u + 1e-4) |P|
* D = rowsum(dO * O) is formed from the forward's bf16 O, whose own error is at most
  u |O| + 2u (|P| |V|) (bf16 rounding of O and of P in the forward):
                                                          D_err   <= sum_c |dO| (u |O| + 2u |P||V|)
* dP is a float32 sum of d exact products:                dP_err  <= d 2^-23 (|dO| |V|^T)
* dS = P (dP - D) is rounded to bf16:                     dS_err  <= (u + 1e-4) |dS| + |P| (D_err + dP_err)
* the three products accumulate n terms in float32:       n 2^-23 times the same sums of magnitudes
so  |dV - dV_ref| <= dP_err^T |dO| + n 2^-23 |P|^T |dO|, and likewise scale (dS_err |K| + ...) for
dQ and scale (dS_err^T |Q| + ...) for dK.  The tests allow twice that bound, plus u |g| when the
gradients are stored as bf16.
"""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200.inputs import normal_dout
from oracle import attention_bwd_chunked_ref, attention_bwd_ref, attention_ref, visible_mask

from gpu_util import device_qkv

pytestmark = pytest.mark.gpu

U = 2.0 ** -9


def _probs_rows(q, k, scale, causal, r0, r1):
    """P for query rows r0..r1-1 of one head (float64, bottom-right causal alignment)."""
    s = scale * (q[r0:r1] @ k.T)
    vis = visible_mask(q.shape[0], k.shape[0], causal)[r0:r1]
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(vis, np.exp(s - m), 0.0)
    den = e.sum(axis=1, keepdims=True)
    return np.divide(e, den, out=np.zeros_like(e), where=den > 0)


def _bounds(q, k, v, do, o_ref, scale, causal, row_chunk=1024):
    """The elementwise bounds of the module docstring for dQ, dK, dV (shapes of q, k, v).

    Evaluated a block of query rows at a time, so that the bench's N = 8192 fits in memory:
    every term of dQ's bound is local to its rows, and dK's and dV's are sums over the rows."""
    shp = [np.shape(x) for x in (q, k, v)]
    q3, k3, v3, do3, o3 = (np.asarray(x, dtype=np.float64).reshape((-1,) + np.shape(x)[-2:])
                           for x in (q, k, v, do, o_ref))
    n, d = q3.shape[1], q3.shape[2]
    acc = n * 2.0 ** -23
    bq, bk, bv = np.zeros_like(q3), np.zeros_like(k3), np.zeros_like(v3)
    for b in range(q3.shape[0]):
        aq, ak, av, ado = np.abs(q3[b]), np.abs(k3[b]), np.abs(v3[b]), np.abs(do3[b])
        for r0 in range(0, n, row_chunk):
            r1 = min(n, r0 + row_chunk)
            p = _probs_rows(q3[b], k3[b], scale, causal, r0, r1)
            dp = do3[b, r0:r1] @ v3[b].T
            ds = p * (dp - (p * dp).sum(-1, keepdims=True))
            ap, ads = np.abs(p), np.abs(ds)
            pv = ap @ av
            d_err = (ado[r0:r1] * (U * np.abs(o3[b, r0:r1]) + 2 * U * pv)).sum(-1)
            dp_err = d * 2.0 ** -23 * (ado[r0:r1] @ av.T)
            ds_err = (U + 1e-4) * ads + ap * (d_err[:, None] + dp_err)
            bv[b] += ((U + 1e-4 + acc) * ap).T @ ado[r0:r1]
            t = ds_err + acc * ads
            bq[b, r0:r1] = scale * (t @ ak)
            bk[b] += scale * (t.T @ aq[r0:r1])
    return bq.reshape(shp[0]), bk.reshape(shp[1]), bv.reshape(shp[2])


def _run(B, H, N, d, causal, g_dtype=torch.float32, seed=0):
    (q, k, v), (tq, tk, tv) = device_qkv(B, H, N, d, seed=seed)
    do = normal_dout(B, H, N, d, seed=seed + 7)
    tdo = torch.from_numpy(do).to(torch.bfloat16).cuda()
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd(tq, tk, tv, causal=causal)  # bf16 O, as the backward expects
    dq, dk, dv = ea.attn_bwd(tq, tk, tv, o, lse, tdo, causal=causal, g_dtype=g_dtype)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    return (q, k, v, do, scale), (dq, dk, dv)


def _check(inputs, grads, causal, bf16_out=False):
    q, k, v, do, scale = inputs
    refs = attention_bwd_ref(q, k, v, do, scale, causal)
    o_ref, _ = attention_ref(q, k, v, scale, causal)
    bounds = _bounds(q, k, v, do, o_ref, scale, causal)
    for name, g, r, b in zip(("dq", "dk", "dv"), grads, refs, bounds):
        g = g.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), name
        tol = 2.0 * b + 1e-6 * np.abs(r).max() + (U * np.abs(r) if bf16_out else 0.0)
        err = np.abs(g - r)
        # a zero bound (the reference and all its terms vanish, e.g. dQ when every row sees at
        # most one key) admits only an exact zero
        assert np.all(err[tol == 0] == 0), name
        worst = float(np.divide(err, tol, out=np.zeros_like(err), where=tol > 0).max())
        assert worst <= 1.0, (name, worst, float(err.max()), float(np.abs(r).max()))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N,d", [
    (1, 1, 128, 64), (1, 2, 256, 128), (2, 1, 384, 64), (1, 1, 1, 128), (1, 1, 7, 64),
    (1, 2, 129, 128), (1, 1, 200, 64), (2, 2, 300, 128), (1, 1, 513, 128),
])
def test_bwd_matches_oracle(B, H, N, d, causal):
    inputs, grads = _run(B, H, N, d, causal)
    _check(inputs, grads, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_bf16_gradients(causal):
    inputs, grads = _run(1, 2, 256, 128, causal, g_dtype=torch.bfloat16, seed=3)
    assert all(g.dtype == torch.bfloat16 for g in grads)
    _check(inputs, grads, causal, bf16_out=True)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_larger_problem(causal):
    inputs, grads = _run(1, 2, 1024, 128, causal, seed=5)
    _check(inputs, grads, causal)


def test_bwd_key_gradients_sum_to_zero():
    """sum_j dK_j = 0 in exact arithmetic; on the GPU it is small against sum_j |dK_j|."""
    inputs, (dq, dk, dv) = _run(1, 2, 512, 128, True, seed=9)
    g = dk.double().cpu().numpy()
    assert np.all(np.abs(g.sum(axis=2)) <= 0.05 * np.abs(g).sum(axis=2) + 1e-6)


def test_bwd_is_deterministic():
    """No atomics: two calls give identical bits."""
    (q, k, v), (tq, tk, tv) = device_qkv(1, 2, 640, 128, seed=11)
    tdo = torch.from_numpy(normal_dout(1, 2, 640, 128, seed=12)).to(torch.bfloat16).cuda()
    o, lse = ea.attn_fwd(tq, tk, tv, causal=True)
    a = ea.attn_bwd(tq, tk, tv, o, lse, tdo, causal=True)
    b = ea.attn_bwd(tq, tk, tv, o, lse, tdo, causal=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bwd_rejects_head_dim_256():
    (q, k, v), (tq, tk, tv) = device_qkv(1, 1, 128, 256)
    o, lse = ea.attn_fwd(tq, tk, tv)
    with pytest.raises(ea.AttnError):
        ea.attn_bwd(tq, tk, tv, o, lse, torch.zeros_like(tq))


def _run_qk(B, H, Nq, Nk, d, causal, seed=0):
    from exact_attention_100_b200.inputs import normal_qkv_lengths
    q, k, v = normal_qkv_lengths(B, H, Nq, Nk, d, seed=seed)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    do = normal_dout(B, H, Nq, d, seed=seed + 7)
    tdo = torch.from_numpy(do).to(torch.bfloat16).cuda()
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd_qk(tq, tk, tv, scale=scale, causal=causal)
    grads = ea.attn_bwd_qk(tq, tk, tv, o, lse, tdo, scale=scale, causal=causal, g_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    return (q, k, v, do, scale), grads


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,Nq,Nk,d", [
    (1, 2, 128, 300, 128), (1, 2, 300, 128, 128), (1, 1, 1, 513, 64), (1, 1, 513, 1, 64),
    (1, 1, 640, 130, 128), (2, 1, 200, 700, 64), (1, 2, 384, 256, 128),
])
def test_bwd_qk_matches_oracle(B, H, Nq, Nk, d, causal):
    """Key length different from the query length; bottom-right causal alignment.  Keys no query
    sees get zero dK, dV; queries that see no key get zero dQ (the oracle's gradients there)."""
    inputs, grads = _run_qk(B, H, Nq, Nk, d, causal)
    _check(inputs, grads, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_qk_equal_lengths_is_attn_bwd(causal):
    (q, k, v), (tq, tk, tv) = device_qkv(1, 2, 333, 128, seed=13)
    tdo = torch.from_numpy(normal_dout(1, 2, 333, 128, seed=14)).to(torch.bfloat16).cuda()
    o, lse = ea.attn_fwd(tq, tk, tv, causal=causal)
    a = ea.attn_bwd(tq, tk, tv, o, lse, tdo, causal=causal)
    b = ea.attn_bwd_qk(tq, tk, tv, o, lse, tdo, causal=causal)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bwd_bench_workload_whole_heads():
    """The workload and call the bench times: B=2 H=16 N=8192 d=128 causal, bf16 O and bf16
    gradients, dO from the recipe (seed 7).  Two whole heads, (0, 0) and (1, 15), against the
    float64 oracle element by element under the bound above (the oracle and the bound taken
    1024 query rows at a time), and a second call bit-identical to the first."""
    B, H, N, d = 2, 16, 8192, 128
    (q, k, v), (tq, tk, tv) = device_qkv(B, H, N, d, seed=0)
    do = normal_dout(B, H, N, d, seed=7)
    tdo = torch.from_numpy(do).to(torch.bfloat16).cuda()
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd(tq, tk, tv, causal=True)
    ws = torch.empty(ea.attn_bwd_workspace_bytes(B, H, N) // 4, dtype=torch.float32, device="cuda")
    g1 = [torch.empty_like(tq) for _ in range(3)]
    g2 = [torch.empty_like(tq) for _ in range(3)]
    ea.attn_bwd(tq, tk, tv, o, lse, tdo, *g1, ws, causal=True)
    ea.attn_bwd(tq, tk, tv, o, lse, tdo, *g2, ws, causal=True)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    for (b, h) in [(0, 0), (1, 15)]:
        sel = lambda x: x[b:b + 1, h:h + 1]
        inputs = (sel(q), sel(k), sel(v), sel(do), scale)
        refs = attention_bwd_chunked_ref(*inputs[:4], scale, True)
        o_ref, _ = attention_ref(*inputs[:3], scale, True)
        bounds = _bounds(*inputs[:4], o_ref, scale, True)
        grads = [g[b:b + 1, h:h + 1].float().cpu().numpy() for g in g1]
        for name, g, r, bd in zip(("dq", "dk", "dv"), grads, refs, bounds):
            g = g.astype(np.float64)
            assert np.isfinite(g).all(), name
            tol = 2.0 * bd + 1e-6 * np.abs(r).max() + U * np.abs(r)
            err = np.abs(g - r)
            assert np.all(err[tol == 0] == 0), name
            worst = float(np.divide(err, tol, out=np.zeros_like(err), where=tol > 0).max())
            assert worst <= 1.0, ((b, h), name, worst, float(err.max()))
