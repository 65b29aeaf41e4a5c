"""Pins for the rotary-embedding oracle (``rope_ref``), CPU only.

Evidence other than the oracle itself: the rotation written as complex multiplication in
float64 (z = (x_i + i x_{i+d/2}) e^{i angle}), exact special angles, invariants of a rotation
(pair norms; the relative-position property of rotary embeddings), torch's float32 CPU ops,
and planted mistakes that these pins must catch.
"""

import numpy as np
import pytest
import torch

from exact_attention_100_b200.inputs import rope_tables
from oracle import hadamard_quant_ref, rope_ref

U32 = 2.0 ** -24  # float32 unit roundoff


def _x(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def _complex_rotation(x, cos, sin):
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape[-2:]
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    w = np.asarray(cos, dtype=np.float64)[:n] + 1j * np.asarray(sin, dtype=np.float64)[:n]
    r = z * w
    return np.concatenate([r.real, r.imag], axis=-1)


def _pins(fn):
    failed = []
    try:
        d, n = 64, 300
        cos, sin = rope_tables(512, d)
        x = _x((2, n, d), 1)
        y = fn(x, cos, sin).astype(np.float64)
        ref = _complex_rotation(x, cos, sin)
        a, b = np.abs(x[..., : d // 2].astype(np.float64)), np.abs(x[..., d // 2:].astype(np.float64))
        c, s = np.abs(cos[:n].astype(np.float64)), np.abs(sin[:n].astype(np.float64))
        mag = np.concatenate([a * c + b * s, b * c + a * s], axis=-1)
        if not np.all(np.abs(y - ref) <= 2 * U32 * (mag + np.abs(ref))):
            failed.append("complex_rotation")
        # position 0 is the identity, a quarter turn maps (a, b) to (-b, a): exactly
        one, zero = np.ones((n, d // 2), np.float32), np.zeros((n, d // 2), np.float32)
        if not np.array_equal(fn(x, one, zero), x):
            failed.append("identity")
        qt = fn(x, zero, one)
        if not np.array_equal(qt, np.concatenate([-x[..., d // 2:], x[..., : d // 2]], axis=-1)):
            failed.append("quarter_turn")
        # relative position: <R_m q, R_n k> = <R_(m-n) q, k> for the angle tables n * theta
        q, k = _x((1, 1, d), 2), _x((1, 1, d), 3)
        for m, nn in [(7, 3), (200, 50), (41, 41)]:
            lhs = np.dot(fn(np.repeat(q, m + 1, 1), cos, sin)[0, m].astype(np.float64),
                         fn(np.repeat(k, nn + 1, 1), cos, sin)[0, nn].astype(np.float64))
            rhs = np.dot(fn(np.repeat(q, m - nn + 1, 1), cos, sin)[0, m - nn].astype(np.float64),
                         k[0, 0].astype(np.float64))
            if abs(lhs - rhs) > 1e-4 * (1 + abs(rhs)):
                failed.append("relative_position")
                break
    except (ValueError, IndexError) as e:
        return ["crash: " + str(e)]
    return failed


def test_oracle_passes_every_pin():
    assert _pins(rope_ref) == []


def test_rotation_preserves_pair_norms():
    d = 128
    cos, sin = rope_tables(256, d)
    x = _x((3, 256, d), 4)
    y = rope_ref(x, cos, sin).astype(np.float64)
    nx = x[..., : d // 2].astype(np.float64) ** 2 + x[..., d // 2:].astype(np.float64) ** 2
    ny = y[..., : d // 2] ** 2 + y[..., d // 2:] ** 2
    assert np.allclose(nx, ny, rtol=1e-6, atol=1e-6)


def test_matches_torch_float32_elementwise_ops():
    """torch's CPU float32 multiply and add/subtract round each operation, in the order stated."""
    d = 128
    cos, sin = rope_tables(200, d)
    x = _x((2, 4, 200, d), 5)
    t = torch.from_numpy(x)
    a, b = t[..., : d // 2], t[..., d // 2:]
    c, s = torch.from_numpy(cos), torch.from_numpy(sin)
    ref = torch.cat([torch.sub(torch.mul(a, c), torch.mul(b, s)), torch.add(torch.mul(b, c), torch.mul(a, s))], -1)
    assert np.array_equal(rope_ref(x, cos, sin), ref.numpy())


def test_fused_preprocessing_is_the_composition():
    """RoPE then H D then per-block E4M3: the quantiser sees the float32 rotated rows exactly."""
    d = 128
    cos, sin = rope_tables(300, d)
    x = np.random.default_rng(6).standard_normal((1, 2, 300, d)).astype(np.float32)
    signs = np.where(np.random.default_rng(7).random(d) < 0.5, -1, 1).astype(np.int8)
    codes, scales = hadamard_quant_ref(rope_ref(x, cos, sin).astype(np.float64), signs)
    # dequantised and un-rotated (H D is orthogonal after normalisation), the rows come back
    from oracle import dequant_ref, hadamard_rotate_ref, sylvester_hadamard
    back = dequant_ref(codes, scales) @ (sylvester_hadamard(d) / np.sqrt(d)) * signs.astype(np.float64)
    rot = rope_ref(x, cos, sin).astype(np.float64)
    assert np.sqrt(np.mean((back - rot) ** 2)) < 0.05 * np.sqrt(np.mean(rot ** 2))
    assert np.allclose(hadamard_rotate_ref(rot, signs) @ (sylvester_hadamard(d) / np.sqrt(d)) * signs, rot)


def _mutant(kind):
    def fn(x, cos, sin):
        x = np.asarray(x, dtype=np.float32)
        n, d = x.shape[-2:]
        c, s = np.asarray(cos, np.float32)[:n], np.asarray(sin, np.float32)[:n]
        if kind == "sin_sign":
            s = -s
        if kind == "cos_sin_swapped":
            c, s = s, c
        if kind == "first_row_only":
            c, s = np.repeat(c[:1], n, 0), np.repeat(s[:1], n, 0)
        if kind == "interleaved":
            a, b = x[..., 0::2], x[..., 1::2]
            out = np.empty_like(x)
            out[..., 0::2] = a * c - b * s
            out[..., 1::2] = b * c + a * s
            return out
        a, b = x[..., : d // 2], x[..., d // 2:]
        return np.concatenate([a * c - b * s, b * c + a * s], axis=-1).astype(np.float32)
    return fn


@pytest.mark.parametrize("kind", ["sin_sign", "cos_sin_swapped", "first_row_only", "interleaved"])
def test_planted_rotation_mistake_is_caught(kind):
    assert _pins(_mutant(kind)) != []
