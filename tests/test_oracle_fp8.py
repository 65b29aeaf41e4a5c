"""Pins for the FP8 pre-processing oracle (CPU only).

The Hadamard pieces are pinned to the textbook (H H^T = d I, Sylvester recursion, scipy's
Hadamard matrix, orthogonality preserving scores); the E4M3 rounding to the OCP format
table in tests/golden/e4m3_values.json and to two library conversions (ml_dtypes and
torch float8_e4m3fn) over every finite bf16 input; the per-block quantiser to its defining
properties.
"""

import json
import math
import os

import ml_dtypes
import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import (E4M3_MAX, dequant_ref, e4m3_decode, e4m3_encode, e4m3_round, fwht_f32,
                    hadamard_quant_ref, hadamard_rotate_ref, sylvester_hadamard, attention_ref)
from exact_attention_100_b200.inputs import hadamard_signs, normal_qkv, round_to_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _all_finite_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    return vals[np.isfinite(vals)]


# ---- Hadamard ------------------------------------------------------------------------------

@pytest.mark.parametrize("d", [1, 2, 4, 64, 128, 256])
def test_sylvester_is_hadamard(d):
    h = sylvester_hadamard(d)
    assert set(np.unique(h)) <= {-1.0, 1.0}
    np.testing.assert_array_equal(h @ h.T, d * np.eye(d))
    np.testing.assert_array_equal(h, scipy.linalg.hadamard(d))


def test_sylvester_h4_explicit():
    assert sylvester_hadamard(4).tolist() == [[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]]


@pytest.mark.parametrize("d", [4, 64, 128, 256])
def test_fwht_matches_matrix(d):
    y = np.random.default_rng(d).standard_normal((9, d)).astype(np.float32)
    got = fwht_f32(y).astype(np.float64)
    want = y.astype(np.float64) @ scipy.linalg.hadamard(d).T
    # float32 butterflies: log2(d) roundings of magnitudes up to sqrt(d) * |y|
    np.testing.assert_allclose(got, want, rtol=0, atol=math.log2(d) * 2 ** -23 * 4 * np.abs(want).max())


def test_fwht_exact_on_small_integers():
    y = np.random.default_rng(3).integers(-50, 50, size=(5, 128)).astype(np.float32)
    np.testing.assert_array_equal(fwht_f32(y).astype(np.float64), y.astype(np.float64) @ scipy.linalg.hadamard(128))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rotation_is_orthogonal_and_keeps_scores(d):
    signs = hadamard_signs(d)
    assert set(np.unique(signs)) == {-1, 1}
    q = np.random.default_rng(1).standard_normal((20, d))
    k = np.random.default_rng(2).standard_normal((30, d))
    qt, kt = hadamard_rotate_ref(q, signs), hadamard_rotate_ref(k, signs)
    np.testing.assert_allclose(qt @ kt.T, q @ k.T, rtol=0, atol=1e-10)
    np.testing.assert_allclose(np.linalg.norm(qt, axis=1), np.linalg.norm(q, axis=1), rtol=1e-13)
    # attention on rotated Q, K is the same attention
    v = np.random.default_rng(3).standard_normal((30, d))
    o1, l1 = attention_ref(q, k, v, 1 / math.sqrt(d), False)
    o2, l2 = attention_ref(qt, kt, v, 1 / math.sqrt(d), False)
    np.testing.assert_allclose(o2, o1, atol=1e-10)
    np.testing.assert_allclose(l2, l1, atol=1e-10)


def test_rotation_spreads_an_outlier():
    d = 128
    x = np.zeros((1, d))
    x[0, 5] = 100.0
    xt = hadamard_rotate_ref(x, hadamard_signs(d))
    np.testing.assert_allclose(np.abs(xt), 100.0 / math.sqrt(d), rtol=1e-14)


# ---- E4M3 ----------------------------------------------------------------------------------

def test_e4m3_golden_table():
    with open(os.path.join(GOLDEN, "e4m3_values.json")) as f:
        g = json.load(f)
    for e in g["values"]:
        assert int(e4m3_encode(e4m3_round(e["value"]))) == e["code"], e
        assert float(e4m3_decode(np.uint8(e["code"]))) == e["value"], e
    for e in g["rounding"]:
        r = float(e4m3_round(e["x"]))
        assert r == e["rounded"] and math.copysign(1, r) == math.copysign(1, e["rounded"]), e


def test_e4m3_all_codes_roundtrip():
    codes = np.arange(256, dtype=np.uint8)
    vals = e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254  # 0x7F and 0xFF are NaN
    np.testing.assert_array_equal(e4m3_encode(vals[finite]), codes[finite])
    np.testing.assert_array_equal(e4m3_round(vals[finite]), vals[finite])
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(vals[finite], lib[finite])
    assert np.nanmax(vals) == E4M3_MAX


def test_e4m3_rounding_matches_libraries_on_every_bf16():
    x = _all_finite_bf16()
    in_range = np.abs(x) < 464.0  # beyond this the libraries return NaN (no saturation)
    xs = x[in_range]
    ours = e4m3_round(xs.astype(np.float64))
    lib1 = xs.astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    lib2 = torch.from_numpy(xs).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, lib1)
    np.testing.assert_array_equal(ours, lib2)
    np.testing.assert_array_equal(np.signbit(ours), np.signbit(lib1))
    big = x[~in_range]
    np.testing.assert_array_equal(e4m3_round(big.astype(np.float64)), np.copysign(E4M3_MAX, big))


def test_e4m3_rounding_matches_library_on_random_float32():
    x = np.random.default_rng(7).standard_normal(200000).astype(np.float32) * np.float32(30)
    x = x[np.abs(x) < 464]
    np.testing.assert_array_equal(e4m3_round(x.astype(np.float64)),
                                  x.astype(ml_dtypes.float8_e4m3fn).astype(np.float64))


# ---- per-block quantiser -------------------------------------------------------------------

@pytest.mark.parametrize("use_hadamard", [False, True])
@pytest.mark.parametrize("n", [1, 128, 300])
def test_block_quant_properties(use_hadamard, n):
    d = 128
    q, _, _ = normal_qkv(2, 3, n, d, seed=5, outlier_frac=0.01)
    signs = hadamard_signs(d) if use_hadamard else None
    codes, scales = hadamard_quant_ref(q, signs)
    nb = (n + 127) // 128
    assert codes.shape == (2, 3, n, d) and codes.dtype == np.uint8
    assert scales.shape == (2, 3, nb) and scales.dtype == np.float32
    vals = e4m3_decode(codes)
    assert not np.any(np.isnan(vals))
    target = hadamard_rotate_ref(q, signs) if use_hadamard else q
    deq = dequant_ref(codes, scales)
    for b in range(2):
        for h in range(3):
            for blk in range(nb):
                r0, r1 = blk * 128, min(n, blk * 128 + 128)
                # the block's largest magnitude lands on (or one rounding from) +-448
                assert np.abs(vals[b, h, r0:r1]).max() >= 416.0
                # element-wise error: half an E4M3 spacing (2^-4 relative) or half a subnormal quantum
                t = target[b, h, r0:r1]
                err = np.abs(deq[b, h, r0:r1] - t)
                s = float(scales[b, h, blk])
                assert np.all(err <= np.abs(t) * 2.0 ** -4 * 1.0001 + s * 2.0 ** -10 * 1.0001 + 1e-6 * np.abs(t))


def test_block_quant_codes_are_scale_invariant_in_powers_of_two():
    q, _, _ = normal_qkv(1, 1, 256, 128, seed=9)
    c1, s1 = hadamard_quant_ref(q, hadamard_signs(128))
    c2, s2 = hadamard_quant_ref(q * 8.0, hadamard_signs(128))
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s2, s1 * np.float32(8))


def test_block_quant_zero_block():
    x = np.zeros((1, 1, 130, 64))
    x[0, 0, 128:] = round_to_bf16(np.random.default_rng(0).standard_normal((2, 64)).astype(np.float32))
    codes, scales = hadamard_quant_ref(x, hadamard_signs(64))
    assert np.all(e4m3_decode(codes[0, 0, :128]) == 0)
    assert scales[0, 0, 0] == np.float32(2.0 ** -126) * np.float32(1 / 8)
    assert np.abs(e4m3_decode(codes[0, 0, 128:])).max() == 448.0


def test_rotation_lowers_block_crest_factor_with_outliers():
    # the transform spreads the outliers: the ratio of a block's largest magnitude to its RMS
    # (what a per-block scale has to cover) drops
    q, _, _ = normal_qkv(1, 2, 512, 128, seed=11, outlier_frac=1e-3)
    qt = hadamard_rotate_ref(q, hadamard_signs(128))
    def crest(x):
        x = x.reshape(-1, 128, 128)
        return np.abs(x).max(axis=(1, 2)) / np.sqrt((x ** 2).mean(axis=(1, 2)))
    assert np.all(crest(qt) < crest(q))
