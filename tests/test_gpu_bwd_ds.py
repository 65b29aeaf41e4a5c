"""GPU parity of attn_bwd_ds, the backward that keeps dS in its workspace (dQ = scale dS K from
the stored tiles instead of recomputing S and dP).

* dQ, dK, dV against the float64 oracle under the elementwise bound derived for attn_bwd (the
  stored dS is the same bf16 dS the dK product uses, so the bound's terms are unchanged);
* dK and dV bit-identical to attn_bwd (the dK/dV kernel's arithmetic is the same; it only
  also stores dS), and two calls bit-identical (no atomics);
* the bench's workload: two whole heads against the oracle.
"""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build
from exact_attention_100_b200.inputs import normal_dout
from gpu_util import device_qkv
from oracle import attention_bwd_chunked_ref, attention_ref
from test_gpu_bwd import U, _bounds, _check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ea_build.build()
    ea.lib()


def _inputs(B, H, N, d, seed):
    (q, k, v), (tq, tk, tv) = device_qkv(B, H, N, d, seed=seed)
    do = normal_dout(B, H, N, d, seed=seed + 7)
    tdo = torch.from_numpy(do).to(torch.bfloat16).cuda()
    return (q, k, v, do), (tq, tk, tv, tdo)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N,d", [
    (1, 1, 128, 64), (1, 2, 256, 128), (2, 1, 384, 64), (1, 1, 1, 128), (1, 1, 7, 64),
    (1, 2, 129, 128), (1, 1, 200, 64), (2, 2, 300, 128), (1, 1, 513, 128),
])
def test_bwd_ds_matches_oracle_and_attn_bwd(B, H, N, d, causal):
    (q, k, v, do), (tq, tk, tv, tdo) = _inputs(B, H, N, d, seed=N + d)
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd(tq, tk, tv, causal=causal)
    g = ea.attn_bwd_ds(tq, tk, tv, o, lse, tdo, causal=causal, g_dtype=torch.float32)
    ref = ea.attn_bwd(tq, tk, tv, o, lse, tdo, causal=causal, g_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    assert torch.equal(g[1], ref[1]) and torch.equal(g[2], ref[2])
    _check((q, k, v, do, scale), g, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_ds_bf16_gradients_and_determinism(causal):
    (q, k, v, do), (tq, tk, tv, tdo) = _inputs(2, 3, 700, 128, seed=5)
    o, lse = ea.attn_fwd(tq, tk, tv, causal=causal)
    ws = torch.empty(ea.attn_bwd_ds_workspace_bytes(2, 3, 700, causal), dtype=torch.uint8, device="cuda")
    g1 = ea.attn_bwd_ds(tq, tk, tv, o, lse, tdo, workspace=ws, causal=causal)
    g2 = ea.attn_bwd_ds(tq, tk, tv, o, lse, tdo, workspace=ws, causal=causal)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    _check((q, k, v, do, 1.0 / math.sqrt(128)), g1, causal, bf16_out=True)


def test_bwd_ds_bench_workload_whole_heads():
    """The bench's backward workload (B=2 H=16 N=8192 d=128 causal, bf16 gradients): two whole
    heads against the float64 oracle under the bound, dK and dV bit-identical to attn_bwd."""
    B, H, N, d = 2, 16, 8192, 128
    (q, k, v, do), (tq, tk, tv, tdo) = _inputs(B, H, N, d, seed=0)
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.attn_fwd(tq, tk, tv, causal=True)
    g = ea.attn_bwd_ds(tq, tk, tv, o, lse, tdo, causal=True)
    ref = ea.attn_bwd(tq, tk, tv, o, lse, tdo, causal=True)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    assert torch.equal(g[1], ref[1]) and torch.equal(g[2], ref[2])
    for (b, h) in [(0, 0), (1, 15)]:
        sel = lambda x: x[b:b + 1, h:h + 1]
        inputs = (sel(q), sel(k), sel(v), sel(do))
        refs = attention_bwd_chunked_ref(*inputs, scale, True)
        o_ref, _ = attention_ref(*inputs[:3], scale, True)
        bounds = _bounds(*inputs, o_ref, scale, True)
        grads = [x[b:b + 1, h:h + 1].float().cpu().numpy() for x in g]
        for name, x, r, bd in zip(("dq", "dk", "dv"), grads, refs, bounds):
            x = x.astype(np.float64)
            assert np.isfinite(x).all(), name
            tol = 2.0 * bd + 1e-6 * np.abs(r).max() + U * np.abs(r)
            err = np.abs(x - r)
            assert np.all(err[tol == 0] == 0), name
            worst = float(np.divide(err, tol, out=np.zeros_like(err), where=tol > 0).max())
            assert worst <= 1.0, ((b, h), name, worst, float(err.max()))


def test_bwd_ds_rejects_what_attn_bwd_rejects():
    (_, (tq, tk, tv, tdo)) = _inputs(1, 1, 256, 128, seed=1)
    o, lse = ea.attn_fwd(tq, tk, tv)
    nbytes = ea.attn_bwd_ds_workspace_bytes(1, 1, 256, False)
    with pytest.raises(ea.AttnError):  # large enough, not 16-byte aligned: the library refuses it
        ea.attn_bwd_ds(tq, tk, tv, o, lse, tdo, workspace=torch.empty(nbytes + 16, dtype=torch.uint8, device="cuda")[1:])
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK


def test_workspace_smaller_than_needed_is_refused_before_any_launch():
    """The C entry points take no workspace size; the binding checks the caller's buffer."""
    (_, (tq, tk, tv, tdo)) = _inputs(1, 2, 300, 64, seed=2)
    o, lse = ea.attn_fwd(tq, tk, tv, causal=True)
    torch.cuda.synchronize()
    launches = ea.attn_num_kernel_launches()
    small_ds = torch.empty(ea.attn_bwd_ds_workspace_bytes(1, 2, 300, True) - 16, dtype=torch.uint8, device="cuda")
    small = torch.empty(ea.attn_bwd_workspace_bytes(1, 2, 300) // 4 - 4, dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        ea.attn_bwd_ds(tq, tk, tv, o, lse, tdo, workspace=small_ds, causal=True)
    with pytest.raises(ValueError):
        ea.attn_bwd(tq, tk, tv, o, lse, tdo, workspace=small, causal=True)
    with pytest.raises(ValueError):
        ea.attn_bwd(tq, tk, tv, o, lse, tdo, workspace=torch.empty(1 << 20, dtype=torch.uint8), causal=True)  # host
    assert ea.attn_num_kernel_launches() == launches
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
