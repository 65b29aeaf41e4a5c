"""Pins for the partial-result merge (``merge_partials_ref``), CPU only: merging the attention of
two disjoint key sets must give the attention of their union (a closed-form identity of the
softmax), for any split, in either order, and with parts that see no key."""

import numpy as np
import pytest

from oracle import attention_ref, merge_partials_ref


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("split", [1, 5, 16, 31])
def test_union_of_key_sets(split):
    q, k, v = _rand((2, 3, 9, 8), 1), _rand((2, 3, 32, 8), 2), _rand((2, 3, 32, 8), 3)
    o, lse = attention_ref(q, k, v, 0.4, False)
    oa, la = attention_ref(q, k[..., :split, :], v[..., :split, :], 0.4, False)
    ob, lb = attention_ref(q, k[..., split:, :], v[..., split:, :], 0.4, False)
    om, lm = merge_partials_ref(oa, la, ob, lb)
    assert np.allclose(om, o, atol=1e-12) and np.allclose(lm, lse, atol=1e-12)
    om2, lm2 = merge_partials_ref(ob, lb, oa, la)  # order does not matter
    assert np.allclose(om2, om, atol=1e-14) and np.allclose(lm2, lm, atol=1e-14)


def test_ring_of_causal_chunks():
    """A causal sequence in 4 chunks: each query chunk merges the full attention of the chunks
    before it and the causal attention of its own chunk -- the whole causal attention."""
    n, c = 40, 10
    q, k, v = _rand((1, 2, n, 4), 4), _rand((1, 2, n, 4), 5), _rand((1, 2, n, 4), 6)
    o, lse = attention_ref(q, k, v, 0.7, True)
    for r in range(4):
        qs = q[..., r * c:(r + 1) * c, :]
        acc_o, acc_l = np.zeros(qs.shape), np.full(qs.shape[:-1], -np.inf)
        for j in range(r + 1):
            ks, vs = k[..., j * c:(j + 1) * c, :], v[..., j * c:(j + 1) * c, :]
            po, pl = attention_ref(qs, ks, vs, 0.7, j == r)
            acc_o, acc_l = merge_partials_ref(acc_o, acc_l, po, pl)
        assert np.allclose(acc_o, o[..., r * c:(r + 1) * c, :], atol=1e-12)
        assert np.allclose(acc_l, lse[..., r * c:(r + 1) * c], atol=1e-12)


def test_parts_without_keys():
    o = _rand((3, 4), 7)
    lse = _rand((3,), 8)
    none_o, none_l = np.zeros((3, 4)), np.full(3, -np.inf)
    for a, b in (((o, lse), (none_o, none_l)), ((none_o, none_l), (o, lse))):
        mo, ml = merge_partials_ref(*a, *b)
        assert np.array_equal(mo, o) and np.array_equal(ml, lse)
    mo, ml = merge_partials_ref(none_o, none_l, none_o, none_l)
    assert np.all(mo == 0) and np.all(np.isneginf(ml))


def test_planted_merge_mistakes_are_caught():
    """Weights by exp(-LSE), or a sum left unnormalised, give the wrong union: each fails the
    union identity (scores of moderate size, so that both parts carry weight)."""
    q, k, v = _rand((1, 1, 6, 4), 9), _rand((1, 1, 12, 4), 10), _rand((1, 1, 12, 4), 11)
    o, lse = attention_ref(q, k, v, 0.5, False)
    oa, la = attention_ref(q, k[..., :5, :], v[..., :5, :], 0.5, False)
    ob, lb = attention_ref(q, k[..., 5:, :], v[..., 5:, :], 0.5, False)

    def wrong_sign(oa, la, ob, lb):
        wa, wb = np.exp(-la), np.exp(-lb)
        return (wa[..., None] * oa + wb[..., None] * ob) / (wa + wb)[..., None], np.log(wa + wb)

    def unnormalised(oa, la, ob, lb):
        m = np.maximum(la, lb)
        wa, wb = np.exp(la - m), np.exp(lb - m)
        return wa[..., None] * oa + wb[..., None] * ob, m + np.log(wa + wb)

    for fn in (wrong_sign, unnormalised):
        mo, ml = fn(oa, la, ob, lb)
        assert not (np.allclose(mo, o, atol=1e-9) and np.allclose(ml, lse, atol=1e-9))
