"""Property-based pins of the float64 oracle (hypothesis, tiny shapes, CPU only).

Each property ties one oracle function to something other than itself over many random shapes:
the pages' tiled recurrence against the two-pass definition for any tile sizes and any pair of
lengths (bottom-right causal), the lazy-rescale variant for any threshold, the merge against the
union of key sets for any split, the packed batch against sequence-by-sequence attention, and
the linearity of attention in V that the definition implies."""

import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import (attention_blockwise_lazy_ref, attention_blockwise_ref, attention_ref, attention_varlen_ref,
                    merge_partials_ref)

SETTINGS = settings(max_examples=40, deadline=None)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@SETTINGS
@given(nq=st.integers(1, 12), nk=st.integers(1, 12), d=st.sampled_from([1, 2, 5, 8]), br=st.integers(1, 7),
       bc=st.integers(1, 7), causal=st.booleans(), seed=st.integers(0, 10 ** 6))
def test_tiled_recurrence_equals_definition(nq, nk, d, br, bc, causal, seed):
    q, k, v = _rand((2, nq, d), seed), _rand((2, nk, d), seed + 1), _rand((2, nk, d), seed + 2)
    o, lse = attention_ref(q, k, v, 0.8, causal)
    ob, lb = attention_blockwise_ref(q, k, v, 0.8, causal, br, bc)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lb))
    assert np.allclose(ob, o, atol=1e-12, rtol=1e-12)
    fin = np.isfinite(lse)
    assert np.allclose(lb[fin], lse[fin], atol=1e-12, rtol=1e-12)


@SETTINGS
@given(n=st.integers(1, 14), d=st.sampled_from([2, 4, 8]), bc=st.integers(1, 6), tau=st.sampled_from([0.0, 1.0, 4.0, 8.0]),
       causal=st.booleans(), seed=st.integers(0, 10 ** 6))
def test_lazy_rescale_equals_definition(n, d, bc, tau, causal, seed):
    q, k, v = _rand((1, n, d), seed) * 3, _rand((1, n, d), seed + 1) * 3, _rand((1, n, d), seed + 2)
    o, lse = attention_ref(q, k, v, 1.0, causal)
    ol, ll = attention_blockwise_lazy_ref(q, k, v, 1.0, causal, bc, tau)
    assert np.allclose(ol, o, atol=1e-10, rtol=1e-10)
    assert np.allclose(ll, lse, atol=1e-10, rtol=1e-10)


@SETTINGS
@given(nq=st.integers(1, 8), nk=st.integers(2, 16), d=st.sampled_from([1, 3, 8]), seed=st.integers(0, 10 ** 6),
       data=st.data())
def test_merge_of_any_split_is_the_union(nq, nk, d, seed, data):
    split = data.draw(st.integers(1, nk - 1))
    q, k, v = _rand((nq, d), seed), _rand((nk, d), seed + 1), _rand((nk, d), seed + 2)
    perm = np.random.default_rng(seed + 3).permutation(nk)  # the two sets need not be contiguous
    a, b = perm[:split], perm[split:]
    o, lse = attention_ref(q, k, v, 0.6, False)
    oa, la = attention_ref(q, k[a], v[a], 0.6, False)
    ob, lb = attention_ref(q, k[b], v[b], 0.6, False)
    om, lm = merge_partials_ref(oa, la, ob, lb)
    assert np.allclose(om, o, atol=1e-12) and np.allclose(lm, lse, atol=1e-12)


@SETTINGS
@given(lens=st.lists(st.tuples(st.integers(0, 6), st.integers(0, 6)), min_size=1, max_size=5),
       causal=st.booleans(), seed=st.integers(0, 10 ** 6))
def test_packed_batch_is_sequence_by_sequence(lens, causal, seed):
    H, d = 2, 3
    cu_q = np.concatenate([[0], np.cumsum([a for a, _ in lens])]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum([b for _, b in lens])]).astype(np.int64)
    q, k, v = _rand((cu_q[-1], H, d), seed), _rand((cu_k[-1], H, d), seed + 1), _rand((cu_k[-1], H, d), seed + 2)
    o, lse = attention_varlen_ref(q, k, v, cu_q, cu_k, 0.9, causal)
    for i, (nq, nk) in enumerate(lens):
        rows = slice(cu_q[i], cu_q[i + 1])
        if nq == 0:
            continue
        if nk == 0:
            assert np.all(o[rows] == 0) and np.all(np.isneginf(lse[:, rows]))
            continue
        keys = slice(cu_k[i], cu_k[i + 1])
        ob, lb = attention_ref(q[rows].transpose(1, 0, 2), k[keys].transpose(1, 0, 2), v[keys].transpose(1, 0, 2),
                               0.9, causal)
        assert np.allclose(o[rows], ob.transpose(1, 0, 2), atol=1e-12)
        fin = np.isfinite(lb)
        assert np.array_equal(np.isneginf(lse[:, rows]), np.isneginf(lb))
        assert np.allclose(lse[:, rows][fin], lb[fin], atol=1e-12)


@SETTINGS
@given(n=st.integers(1, 10), d=st.sampled_from([1, 4, 7]), alpha=st.floats(-3, 3), causal=st.booleans(),
       seed=st.integers(0, 10 ** 6))
def test_output_is_affine_in_v(n, d, alpha, causal, seed):
    """O(V alpha + 1 c^T) = alpha O(V) + 1 c^T: each output row is a convex combination of V rows,
    and the LSE does not depend on V."""
    q, k, v = _rand((n, d), seed), _rand((n, d), seed + 1), _rand((n, d), seed + 2)
    c = _rand((d,), seed + 3)
    o, lse = attention_ref(q, k, v, 0.5, causal)
    o2, lse2 = attention_ref(q, k, alpha * v + c, 0.5, causal)
    assert np.allclose(o2, alpha * o + c, atol=1e-12)
    assert np.array_equal(lse, lse2)
