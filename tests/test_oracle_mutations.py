"""Planted mistakes: each plausible slip in the oracle must fail at least one pin.

The mutants below are copies of the oracle's arithmetic with one mistake planted (a dropped
scale, an off-by-one causal mask, the softmax over the wrong axis, a transposed operand, a
dropped LSE term, ties rounded away from zero, a wrong butterfly sign).  The pin checks are
the same kinds of evidence the oracle's own tests use.  CPU only.
"""

import json
import math
import os

import ml_dtypes
import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import attention_ref, e4m3_round, fwht_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _mutant_attention(mutation):
    def fn(q, k, v, scale, causal):
        q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
        if mutation == "no_scale":
            scale = 1.0
        kk = k
        if mutation == "q_for_k":
            kk = q
        s = scale * (q @ kk.swapaxes(-1, -2))
        n_q, n_k = s.shape[-2:]
        i = np.arange(n_q)[:, None]
        j = np.arange(n_k)[None, :]
        if causal:
            vis = (j < i) | ((i == 0) & (j == 0)) if mutation == "strict_causal" else j <= i
            s = np.where(vis, s, -np.inf)
        axis = -2 if mutation == "wrong_axis" else -1
        m = s.max(axis=axis, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=axis, keepdims=True)
        p = e / l
        o = p @ v
        if mutation == "lse_no_max":
            lse = np.log(l)[..., 0] if axis == -1 else np.log(l)[..., 0, :]
        else:
            lse = (m + np.log(l))[..., 0] if axis == -1 else (m + np.log(l))[..., 0, :]
        return o, lse
    return fn


def _pins_attention(fn):
    """Returns the list of pin names the function fails (a crash fails every pin)."""
    try:
        return _pins_attention_inner(fn)
    except (ValueError, IndexError) as e:
        return ["crash: " + str(e)]


def _pins_attention_inner(fn):
    failed = []
    with open(os.path.join(GOLDEN, "attention_handworked.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        o, lse = fn(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]), c["scale"], c["causal"])
        if not (np.allclose(o, c["o"], atol=1e-9) and np.allclose(lse, c["lse"], atol=1e-9)):
            failed.append("handworked:" + c["name"])
    rng = np.random.default_rng(0)
    for causal in (False, True):
        q, k, v = (rng.standard_normal((2, 40, 16)) for _ in range(3))
        qt, kt, vt = (torch.from_numpy(t) for t in (q, k, v))
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=0.25).numpy()
        o, _ = fn(q, k, v, 0.25, causal)
        if not np.allclose(o, ref, atol=1e-10):
            failed.append(f"sdpa(causal={causal})")
    q, k, v = (rng.standard_normal((30, 8)) for _ in range(3))
    o, lse = fn(q, k, v, 0.5, True)
    if not np.allclose(o[0], v[0], atol=1e-12):
        failed.append("causal_row0")
    s = 0.5 * q @ k.T
    tot = np.array([np.exp(s[i, : i + 1]).sum() for i in range(30)])
    if not np.allclose(np.exp(lse), tot, rtol=1e-10):
        failed.append("exp_sum_lse")
    return failed


def test_real_oracle_passes_every_pin():
    assert _pins_attention(lambda q, k, v, s, c: attention_ref(q, k, v, s, c)) == []
    assert _pins_attention(_mutant_attention("none")) == []


@pytest.mark.parametrize("mutation", ["no_scale", "strict_causal", "wrong_axis", "q_for_k", "lse_no_max"])
def test_planted_attention_mistake_is_caught(mutation):
    assert _pins_attention(_mutant_attention(mutation)), mutation


def _round_half_away(x):
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    quantum = np.where(a < 2.0 ** -6, 2.0 ** -9, np.ldexp(1.0, ex - 1 - 3))
    r = np.minimum(np.floor(a / quantum + 0.5) * quantum, 448.0)
    return np.copysign(r, x)


def _pins_e4m3(fn):
    bits = np.arange(1 << 16, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) < 464)]
    return not np.array_equal(fn(x.astype(np.float64)), x.astype(ml_dtypes.float8_e4m3fn).astype(np.float64))


def test_planted_rounding_mistake_is_caught():
    assert not _pins_e4m3(e4m3_round)
    assert _pins_e4m3(_round_half_away)


def _fwht_wrong_sign(y):
    y = np.array(y, dtype=np.float32)
    d = y.shape[-1]
    h = 1
    while h < d:
        t = y.reshape(y.shape[:-1] + (d // (2 * h), 2, h))
        a, b = t[..., 0, :], t[..., 1, :]
        y = np.stack([a + b, b - a] if h == 4 else [a + b, a - b], axis=-2).reshape(y.shape)
        h *= 2
    return y


def test_planted_butterfly_mistake_is_caught():
    y = np.random.default_rng(1).integers(-9, 9, size=(3, 64)).astype(np.float32)
    want = y.astype(np.float64) @ scipy.linalg.hadamard(64)
    assert np.array_equal(fwht_f32(y), want)
    assert not np.array_equal(_fwht_wrong_sign(y), want)
