"""Pins of the backward oracle (``oracle.attention_bwd``), CPU only.

The pages print no gradient and no worked example, so the pins are what the mathematics
fixes: central finite differences of the *forward* oracle (a different computation: two
passes with a row max), torch float64 autograd through the forward formula, and invariants
of the softmax Jacobian.  A planted-mistake suite at the end shows that each plausible slip
fails one of them.
"""

import numpy as np
import pytest
import torch

from oracle import attention_bwd_ref, attention_ref, softmax_bwd_delta, softmax_probs


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _fd_grads(q, k, v, do, scale, causal, h=1e-6):
    """Central differences of L = sum(dO * O) through the forward oracle."""
    def loss(qq, kk, vv):
        o, _ = attention_ref(qq, kk, vv, scale, causal)
        return float(np.sum(do * o))

    grads = []
    for which in range(3):
        base = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(base[which])
        it = np.nditer(base[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [t.copy() for t in base]
            minus = [t.copy() for t in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(5, 3), (8, 4), (9, 2)])
def test_matches_finite_differences_of_forward_oracle(causal, n, d):
    q, k, v, do = (_rand((1, n, d), s) for s in (1, 2, 3, 4))
    scale = 0.7
    ref = attention_bwd_ref(q, k, v, do, scale, causal)
    fd = _fd_grads(q, k, v, do, scale, causal)
    for a, b in zip(ref, fd):
        np.testing.assert_allclose(a, b, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_autograd_float64(causal):
    b, h, n, d = 2, 3, 37, 16
    q, k, v, do = (_rand((b, h, n, d), s) for s in (5, 6, 7, 8))
    scale = d ** -0.5
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    o.backward(torch.tensor(do))
    ref = attention_bwd_ref(q, k, v, do, scale, causal)
    for a, t in zip(ref, (tq, tk, tv)):
        np.testing.assert_allclose(a, t.grad.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_delta_identity(causal):
    """rowsum(P * dP) equals rowsum(dO * O): the form a tiled kernel computes up front."""
    q, k, v, do = (_rand((2, 23, 8), s) for s in (9, 10, 11, 12))
    scale = 0.4
    p = softmax_probs(q, k, scale, causal)
    dp = np.einsum("bic,bjc->bij", do, v)
    o, _ = attention_ref(q, k, v, scale, causal)
    np.testing.assert_allclose((p * dp).sum(-1), softmax_bwd_delta(o, do), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_key_gradients_sum_to_zero(causal):
    """Each row of dS sums to zero (softmax Jacobian), so sum_j dK_j = 0 exactly."""
    q, k, v, do = (_rand((3, 31, 8), s) for s in (13, 14, 15, 16))
    _, dk, _ = attention_bwd_ref(q, k, v, do, 0.5, causal)
    np.testing.assert_allclose(dk.sum(axis=-2), 0.0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_value_gradients_sum_to_output_gradients(causal):
    """Rows of P sum to one, so sum_j dV_j = sum_i dO_i."""
    q, k, v, do = (_rand((2, 19, 6), s) for s in (17, 18, 19, 20))
    _, _, dv = attention_bwd_ref(q, k, v, do, 0.3, causal)
    np.testing.assert_allclose(dv.sum(axis=-2), do.sum(axis=-2), rtol=1e-12, atol=1e-12)


def test_identical_keys_give_zero_query_gradient():
    """With every key equal, dQ_i = scale * k * sum_j dS_ij = 0."""
    q, v, do = (_rand((1, 12, 5), s) for s in (21, 22, 23))
    k = np.repeat(_rand((1, 1, 5), 24), 12, axis=1)
    dq, _, _ = attention_bwd_ref(q, k, v, do, 0.9, False)
    np.testing.assert_allclose(dq, 0.0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_shifting_values_leaves_q_and_k_gradients(causal):
    """V -> V + c (one vector added to every row) shifts O by c: dQ and dK do not change."""
    q, k, v, do = (_rand((1, 17, 4), s) for s in (25, 26, 27, 28))
    c = _rand((1, 1, 4), 29)
    a = attention_bwd_ref(q, k, v, do, 0.6, causal)
    b = attention_bwd_ref(q, k, v + c, do, 0.6, causal)
    np.testing.assert_allclose(a[0], b[0], atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], atol=1e-12)


def test_causal_first_row_gradient():
    """Causal row 0 sees only key 0: O_0 = v_0, so dV_0 gets dO_0 in full from row 0 and
    dQ_0 = 0 (a one-element softmax has zero Jacobian)."""
    q, k, v, do = (_rand((1, 6, 3), s) for s in (30, 31, 32, 33))
    dq, _, _ = attention_bwd_ref(q, k, v, do, 1.0, True)
    np.testing.assert_allclose(dq[0, 0], 0.0, atol=1e-14)


# ----------------------------------------------------------------------------- planted mistakes
def _mutant_bwd(mutation):
    def fn(q, k, v, do, scale, causal):
        p = softmax_probs(q, k, scale, causal)
        if mutation == "strict_causal" and causal:
            n = p.shape[-1]
            mask = np.tril(np.ones((n, n)), -1) + np.eye(n) * (np.arange(n) == 0)
            p = p * mask
            p = p / np.maximum(p.sum(-1, keepdims=True), 1e-300)
        dv = np.einsum("bji,bic->bjc" if mutation == "p_not_transposed" else "bij,bic->bjc", p, do)
        dp = np.einsum("bic,bjc->bij", do, v)
        if mutation == "no_delta":
            ds = p * dp
        elif mutation == "delta_from_v":
            ds = p * (dp - np.einsum("bic,bic->bi", do, v[:, : do.shape[1]])[..., None])
        else:
            ds = p * (dp - (p * dp).sum(axis=-1, keepdims=True))
        sq = 1.0 if mutation == "no_scale_dq" else scale
        dq = sq * np.einsum("bij,bjc->bic", ds, k)
        dk = scale * np.einsum("bji,bic->bjc" if mutation == "ds_not_transposed" else "bij,bic->bjc", ds, q)
        return dq, dk, dv
    return fn


def _pins_pass(fn):
    """The pins above, run against a candidate backward; False as soon as one fails."""
    try:
        for causal in (False, True):
            q, k, v, do = (_rand((1, 7, 3), s) for s in (41, 42, 43, 44))
            got = fn(q, k, v, do, 0.8, causal)
            fd = _fd_grads(q, k, v, do, 0.8, causal)
            for a, b in zip(got, fd):
                if not np.allclose(a, b, rtol=1e-6, atol=1e-8):
                    return False
            if not np.allclose(got[1].sum(axis=-2), 0.0, atol=1e-10):
                return False
            if not np.allclose(got[2].sum(axis=-2), do.sum(axis=-2), atol=1e-10):
                return False
        return True
    except Exception:
        return False


def test_pins_accept_the_oracle():
    assert _pins_pass(lambda q, k, v, do, s, c: attention_bwd_ref(q, k, v, do, s, c))


@pytest.mark.parametrize("mutation", ["no_delta", "delta_from_v", "p_not_transposed", "no_scale_dq",
                                      "ds_not_transposed", "strict_causal"])
def test_planted_mistake_fails_a_pin(mutation):
    assert not _pins_pass(_mutant_bwd(mutation))


# ---- the row-chunked backward (used at sizes whose score matrix does not fit in memory) -------

from oracle import attention_bwd_chunked_ref  # noqa: E402


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk,chunk", [(37, 37, 1), (37, 37, 5), (40, 23, 7), (23, 40, 16), (64, 64, 64),
                                         (50, 50, 1024)])
def test_chunked_backward_equals_whole_matrix(nq, nk, chunk, causal):
    """Query-row blocks of any size (dividing N or not, longer than N) give the whole-matrix
    gradients: dQ rows are local to their block, dK and dV are sums over the blocks."""
    rng = np.random.default_rng(nq * 100 + nk + chunk)
    q, k, v = (rng.standard_normal((2, n, 16)) for n in (nq, nk, nk))
    do = rng.standard_normal((2, nq, 16))
    a = attention_bwd_ref(q, k, v, do, 0.3, causal)
    b = attention_bwd_chunked_ref(q, k, v, do, 0.3, causal, row_chunk=chunk)
    for x, y in zip(a, b):
        assert x.shape == y.shape
        assert np.abs(x - y).max() <= 1e-12 * max(1.0, np.abs(x).max())


def test_chunked_backward_matches_finite_differences():
    """Independently of the whole-matrix form: central differences of the forward oracle."""
    q, k, v = (_rand((1, 9, 4), s) for s in (31, 32, 33))
    do = _rand((1, 9, 4), 34)
    got = attention_bwd_chunked_ref(q, k, v, do, 0.7, True, row_chunk=4)
    for g, r in zip(got, _fd_grads(q, k, v, do, 0.7, True)):
        assert np.abs(g - r).max() <= 1e-6


def test_chunked_backward_planted_mistake_fails():
    """dV taken from the last block only (assigned, not summed) must fail the equality pin."""
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((1, 30, 8)) for _ in range(3))
    do = rng.standard_normal((1, 30, 8))
    ref = attention_bwd_ref(q, k, v, do, 0.5, False)[2]
    wrong = np.zeros_like(v)
    for r0 in range(0, 30, 7):
        p = softmax_probs(q[:, r0:r0 + 7], k, 0.5, False)
        wrong[0] = p[0].T @ do[0, r0:r0 + 7]
    assert np.abs(wrong - ref).max() > 1e-3
