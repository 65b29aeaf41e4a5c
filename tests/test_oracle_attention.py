"""Pins for the float64 attention oracle (CPU only).

Each check ties the oracle to something other than itself: hand-worked instances of the
definition, closed forms, invariants that any correct softmax attention satisfies, an
independent algorithm (the pages' blockwise recurrence) and a library routine (torch's
scaled_dot_product_attention evaluated in float64 on the CPU).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention_blockwise_lazy_ref, attention_blockwise_ref, attention_ref, visible_mask
from exact_attention_100_b200.inputs import normal_qkv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---- hand-worked instances of the definition -------------------------------------------

def test_handworked_cases():
    with open(os.path.join(GOLDEN, "attention_handworked.json")) as f:
        cases = json.load(f)["cases"]
    env = {"log": math.log, "exp": math.exp}
    for c in cases:
        # the stored numbers are the closed forms (guards against a typo in the fixture)
        for row, row_cf in zip(c["o"], c["o_closed_form"]):
            for x, cf in zip(row, row_cf):
                assert x == pytest.approx(eval(cf, env), abs=1e-15), c["name"]
        for x, cf in zip(c["lse"], c["lse_closed_form"]):
            assert x == pytest.approx(eval(cf, env), abs=1e-15), c["name"]
        o, lse = attention_ref(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]),
                               c["scale"], c["causal"])
        np.testing.assert_allclose(o, np.array(c["o"]), rtol=0, atol=1e-12, err_msg=c["name"])
        np.testing.assert_allclose(lse, np.array(c["lse"]), rtol=0, atol=1e-12, err_msg=c["name"])


# ---- closed forms ------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_visible_values(causal):
    n, d = 37, 8
    q = _rand((n, d), 1)
    k = np.tile(_rand((1, d), 2), (n, 1))
    v = _rand((n, d), 3)
    scale = 1 / math.sqrt(d)
    o, lse = attention_ref(q, k, v, scale, causal)
    s = scale * (q @ k[0])  # every score of row i equals s_i
    for i in range(n):
        nvis = i + 1 if causal else n
        np.testing.assert_allclose(o[i], v[:nvis].mean(axis=0), rtol=0, atol=1e-12)
        assert lse[i] == pytest.approx(s[i] + math.log(nvis), abs=1e-12)


def test_dominant_score_selects_that_value_row():
    n, d = 50, 16
    rng = np.random.default_rng(4)
    q = rng.standard_normal((n, d)) * 0.01
    k = rng.standard_normal((n, d)) * 0.01
    v = rng.standard_normal((n, d))
    jstar = rng.integers(0, n, size=n)
    # one-hot extra coordinates: score(i, j) = (tiny) + 60 * [j == jstar[i]]
    q = np.hstack([q, 60.0 * np.eye(n)[jstar]])
    k = np.hstack([k, np.eye(n)])
    o, _ = attention_ref(q, k, v, 1.0, False)
    # every other weight is below exp(-59.9); their total below n * exp(-59.9)
    np.testing.assert_allclose(o, v[jstar], rtol=0, atol=n * math.exp(-59.9) * np.abs(v).max() * 2)


def test_causal_row0_is_v0():
    q, k, v = (_rand((3, 64, 32), s) for s in (5, 6, 7))
    o, lse = attention_ref(q, k, v, 0.3, True)
    np.testing.assert_allclose(o[:, 0], v[:, 0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[:, 0], 0.3 * np.einsum("bd,bd->b", q[:, 0], k[:, 0]), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_values_pass_through(causal):
    q, k = _rand((40, 8), 8), _rand((40, 8), 9)
    v = np.full((40, 8), -2.5)
    o, _ = attention_ref(q, k, v, 0.7, causal)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-13)


# ---- invariants --------------------------------------------------------------------------

def test_joint_kv_permutation_invariance_noncausal():
    q, k, v = (_rand((2, 70, 16), s) for s in (10, 11, 12))
    perm = np.random.default_rng(13).permutation(70)
    o1, l1 = attention_ref(q, k, v, 0.25, False)
    o2, l2 = attention_ref(q, k[:, perm], v[:, perm], 0.25, False)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_exp_sum_equals_exp_lse(causal):
    q, k, v = (_rand((33, 24), s) for s in (14, 15, 16))
    scale = 1 / math.sqrt(24)
    _, lse = attention_ref(q, k, v, scale, causal)
    vis = visible_mask(33, 33, causal)
    for i in range(33):
        s = scale * (k @ q[i])
        tot = sum(math.exp(s[j]) for j in range(33) if vis[i, j])  # plain Python loop
        assert math.exp(lse[i]) == pytest.approx(tot, rel=1e-12)


def test_rows_are_convex_combinations():
    q, k, v = (_rand((1, 2, 90, 8), s) for s in (17, 18, 19))
    o, _ = attention_ref(q, k, v, 1.3, False)
    assert np.all(o <= v.max(axis=-2, keepdims=True) + 1e-12)
    assert np.all(o >= v.min(axis=-2, keepdims=True) - 1e-12)


def test_row_chunking_does_not_change_result():
    q, k, v = (_rand((2, 300, 16), s) for s in (20, 21, 22))
    a = attention_ref(q, k, v, 0.2, True, row_chunk=1024)
    b = attention_ref(q, k, v, 0.2, True, row_chunk=7)
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-14)


def test_causal_mask_bottom_right_alignment():
    m = visible_mask(2, 4, True)
    assert m.tolist() == [[True, True, True, False], [True, True, True, True]]
    assert visible_mask(3, 3, True).tolist() == [[True, False, False], [True, True, False], [True, True, True]]


def test_fully_masked_row_convention():
    # only reachable with more queries than keys: row 0 then sees no key
    q, k, v = _rand((3, 4), 23), _rand((2, 4), 24), _rand((2, 4), 25)
    o, lse = attention_ref(q, k, v, 1.0, True)
    assert np.all(o[0] == 0) and lse[0] == -np.inf
    np.testing.assert_allclose(o[1], v[0], atol=1e-14)


# ---- library routine: torch SDPA in float64 on the CPU ------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 64), (127, 64), (200, 128), (64, 256)])
def test_matches_torch_sdpa_float64(causal, n, d):
    q, k, v = (torch.from_numpy(_rand((2, 3, n, d), s)) for s in (26, 27, 28))
    scale = 1 / math.sqrt(d)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=scale)
    s = scale * q @ k.transpose(-1, -2)
    if causal:
        s = s.masked_fill(~torch.ones(n, n, dtype=torch.bool).tril(), float("-inf"))
    ref_lse = torch.logsumexp(s, dim=-1)
    o, lse = attention_ref(q.numpy(), k.numpy(), v.numpy(), scale, causal)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


# ---- independent algorithm: the pages' blockwise recurrence -------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 4), (17, 8), (64, 64), (45, 4)])
@pytest.mark.parametrize("bc", [1, 3, 16, 64])
def test_blockwise_equals_two_pass(causal, n, d, bc):
    q, k, v = (_rand((2, n, d), s) for s in (29, 30, 31))
    for br in (1, 5, n):
        o1, l1 = attention_ref(q, k, v, 1 / math.sqrt(d), causal)
        o2, l2 = attention_blockwise_ref(q, k, v, 1 / math.sqrt(d), causal, br, bc)
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.0, 1.0, 8.0, 1e9])
@pytest.mark.parametrize("bc", [1, 7, 32])
def test_lazy_rescale_recurrence_is_exact(causal, tau, bc):
    q, k, v = (_rand((2, 61, 16), s) * 2.0 for s in (32, 33, 34))
    o1, l1 = attention_ref(q, k, v, 0.4, causal)
    o2, l2 = attention_blockwise_lazy_ref(q, k, v, 0.4, causal, bc, tau)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-11)


def test_on_seeded_bf16_workload_small_config():
    # the small parity configuration: B=1 H=1 N=256 d=64, seed 0
    q, k, v = normal_qkv(1, 1, 256, 64, seed=0)
    o1, l1 = attention_ref(q, k, v, 1 / 8.0, False)
    o2, l2 = attention_blockwise_ref(q, k, v, 1 / 8.0, False, 128, 128)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)
    assert np.all(np.isfinite(o1)) and o1.shape == (1, 1, 256, 64)
