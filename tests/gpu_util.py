"""Helpers shared by the GPU parity tests: seeded inputs on the device and comparisons with the
float64 oracle (whole outputs for small problems, sampled rows for large ones)."""

from __future__ import annotations

import math

import numpy as np

from oracle import attention_ref
from exact_attention_100_b200.inputs import normal_qkv

# Tolerances for bf16 inputs ~ N(0,1) against the float64 oracle (the bar the spec sets):
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_REL = 1e-3


def device_qkv(B, H, N, d, seed=0, **kw):
    import torch
    q, k, v = normal_qkv(B, H, N, d, seed=seed, **kw)
    to = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda()  # exact: values are bf16 already
    return (q, k, v), (to(q), to(k), to(v))


def compare_full(o_gpu, lse_gpu, q, k, v, scale, causal):
    o_ref, lse_ref = attention_ref(q, k, v, scale, causal)
    o = o_gpu.float().cpu().numpy().astype(np.float64)
    lse = lse_gpu.cpu().numpy().astype(np.float64)
    err = np.abs(o - o_ref)
    lse_rel = np.abs(lse - lse_ref) / np.maximum(np.abs(lse_ref), 1e-30)
    return dict(o_max_abs=float(err.max()), o_mean_abs=float(err.mean()), lse_max_rel=float(lse_rel.max()),
                finite=bool(np.isfinite(o).all() and np.isfinite(lse).all()))


def sampled_rows(B, H, N, n_rows, seed=123):
    """(b, h, i) triples: first and last rows of the sequence plus random ones."""
    rng = np.random.default_rng(seed)
    rows = [(0, 0, 0), (B - 1, H - 1, N - 1), (0, H - 1, min(N - 1, 127)), (B - 1, 0, min(N - 1, 128))]
    for _ in range(n_rows - len(rows)):
        rows.append((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))))
    return rows


def compare_rows(o_gpu, lse_gpu, q, k, v, scale, causal, rows):
    """Oracle one row at a time: row i of a causal problem is the non-causal problem on keys 0..i."""
    errs, lrel = [], []
    o_cpu = {}
    for (b, h, i) in rows:
        lim = i + 1 if causal else k.shape[2]
        o_ref, lse_ref = attention_ref(q[b, h, i:i + 1], k[b, h, :lim], v[b, h, :lim], scale, False)
        key = (b, h)
        if key not in o_cpu:
            o_cpu[key] = (o_gpu[b, h].float().cpu().numpy(), lse_gpu[b, h].cpu().numpy())
        og, lg = o_cpu[key]
        errs.append(np.abs(og[i].astype(np.float64) - o_ref[0]))
        lrel.append(abs(float(lg[i]) - lse_ref[0]) / max(abs(lse_ref[0]), 1e-30))
    e = np.stack(errs)
    return dict(o_max_abs=float(e.max()), o_mean_abs=float(e.mean()), lse_max_rel=float(max(lrel)))


def assert_within(res, what=""):
    assert res.get("finite", True), (what, res)
    assert res["o_max_abs"] <= O_MAX_ABS, (what, res)
    assert res["o_mean_abs"] <= O_MEAN_ABS, (what, res)
    assert res["lse_max_rel"] <= LSE_REL, (what, res)


def default_scale(d):
    return 1.0 / math.sqrt(d)
