"""Pins for the packed variable-length oracle (``attention_varlen_ref``), CPU only.

The packed batch is a bookkeeping layer over the definition, so its pins check the
bookkeeping against things other than itself: a brute-force evaluation of the definition with
scalar Python loops over every row of a tiny packed batch (lengths 0, 1, more queries than keys,
more keys than queries), the fixed-length oracle on a batch of equal lengths, independence of
the sequences, and planted mistakes that these pins must catch.
"""

import math

import numpy as np
import pytest

from oracle import attention_ref, attention_varlen_ref

# (Nq_b, Nk_b) per sequence: an empty query sequence, an empty key sequence, one key, more
# queries than keys (causal rows with no key), more keys than queries
LENGTHS = [(3, 5), (0, 2), (2, 0), (4, 1), (5, 3), (1, 6)]


def _packed(lengths, H, d, seed):
    rng = np.random.default_rng(seed)
    cu_q = np.concatenate([[0], np.cumsum([a for a, _ in lengths])]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum([b for _, b in lengths])]).astype(np.int64)
    q = rng.standard_normal((cu_q[-1], H, d))
    k = rng.standard_normal((cu_k[-1], H, d))
    v = rng.standard_normal((cu_k[-1], H, d))
    return q, k, v, cu_q, cu_k


def _brute(q, k, v, cu_q, cu_k, scale, causal):
    """The definition row by row with scalar loops: softmax over the visible keys of the row's
    own sequence, bottom-right aligned (key j visible to query i iff j <= i + Nk - Nq)."""
    total_q, H, d = q.shape
    out = np.zeros((total_q, H, d))
    lse = np.full((H, total_q), -math.inf)
    for b in range(len(cu_q) - 1):
        nq, nk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        for h in range(H):
            for i in range(nq):
                vis = [j for j in range(nk) if not causal or j <= i + nk - nq]
                if not vis:
                    continue
                s = {j: scale * sum(q[cu_q[b] + i, h, c] * k[cu_k[b] + j, h, c] for c in range(d)) for j in vis}
                m = max(s.values())
                w = {j: math.exp(s[j] - m) for j in vis}
                z = sum(w.values())
                for c in range(d):
                    out[cu_q[b] + i, h, c] = sum(w[j] * v[cu_k[b] + j, h, c] for j in vis) / z
                lse[h, cu_q[b] + i] = m + math.log(z)
    return out, lse


def _pins(fn):
    """Names of the pins that ``fn`` fails (a crash fails them all)."""
    failed = []
    try:
        for causal in (False, True):
            q, k, v, cu_q, cu_k = _packed(LENGTHS, 2, 4, seed=1)
            o, lse = fn(q, k, v, cu_q, cu_k, 0.7, causal)
            ob, lb = _brute(q, k, v, cu_q, cu_k, 0.7, causal)
            if not (np.allclose(o, ob, atol=1e-12, rtol=0) and np.array_equal(np.isneginf(lse), np.isneginf(lb))
                    and np.allclose(lse[np.isfinite(lb)], lb[np.isfinite(lb)], atol=1e-12, rtol=0)):
                failed.append("brute_force_%d" % causal)
            # equal lengths: the fixed-length oracle on the unpacked batch
            B, H, N, d = 3, 2, 7, 5
            rng = np.random.default_rng(3)
            qb, kb, vb = (rng.standard_normal((B, H, N, d)) for _ in range(3))
            pack = lambda x: x.transpose(0, 2, 1, 3).reshape(B * N, H, d)
            cu = np.arange(B + 1) * N
            o, lse = fn(pack(qb), pack(kb), pack(vb), cu, cu, 0.4, causal)
            of, lf = attention_ref(qb, kb, vb, 0.4, causal)
            if not (np.allclose(o, pack(of), atol=1e-12, rtol=0)
                    and np.allclose(lse, lf.transpose(1, 0, 2).reshape(H, B * N), atol=1e-12, rtol=0)):
                failed.append("equal_lengths_%d" % causal)
    except (ValueError, IndexError) as e:
        return ["crash: " + str(e)]
    return failed


def test_oracle_passes_every_pin():
    assert _pins(attention_varlen_ref) == []


def test_sequences_are_independent():
    q, k, v, cu_q, cu_k = _packed(LENGTHS, 2, 8, seed=4)
    o, lse = attention_varlen_ref(q, k, v, cu_q, cu_k, 0.5, True)
    # change every row of sequence 4 (queries and keys): other sequences' results are unchanged
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[cu_q[4]:cu_q[5]] += 3.0
    k2[cu_k[4]:cu_k[5]] *= -2.0
    v2[cu_k[4]:cu_k[5]] += 7.0
    o2, lse2 = attention_varlen_ref(q2, k2, v2, cu_q, cu_k, 0.5, True)
    keep = np.ones(cu_q[-1], dtype=bool)
    keep[cu_q[4]:cu_q[5]] = False
    assert np.array_equal(o[keep], o2[keep]) and np.array_equal(lse[:, keep], lse2[:, keep])
    assert not np.array_equal(o[~keep], o2[~keep])


def test_empty_key_sequence_gives_zero_and_minus_inf():
    q, k, v, cu_q, cu_k = _packed(LENGTHS, 3, 4, seed=5)
    for causal in (False, True):
        o, lse = attention_varlen_ref(q, k, v, cu_q, cu_k, 1.0, causal)
        rows = slice(cu_q[2], cu_q[3])  # sequence 2 has 2 queries and no keys
        assert np.all(o[rows] == 0) and np.all(np.isneginf(lse[:, rows]))


def _mutant(kind):
    def fn(q, k, v, cu_q, cu_k, scale, causal):
        total_q, H, _ = q.shape
        out = np.zeros((total_q, H, v.shape[2]))
        lse = np.full((H, total_q), -np.inf)
        for b in range(len(cu_q) - 1):
            q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
            kc = cu_q if kind == "query_offsets_for_keys" else cu_k
            k0, k1 = int(kc[b]), int(kc[b + 1])
            if kind == "one_row_short":
                q1 = max(q0, q1 - 1)
            if q1 == q0 or k1 == k0:
                continue
            qs, ks, vs = (x.transpose(1, 0, 2) for x in (q[q0:q1], k[k0:k1], v[k0:k1]))
            if kind == "top_left_causal" and causal:
                nq, nk = q1 - q0, k1 - k0
                s = scale * qs @ ks.transpose(0, 2, 1)
                s = np.where(np.arange(nk)[None, :] <= np.arange(nq)[:, None], s, -np.inf)
                m = s.max(-1, keepdims=True)
                m = np.where(np.isfinite(m), m, 0.0)
                e = np.exp(s - m)
                z = e.sum(-1, keepdims=True)
                o_b = np.where(z > 0, (e / np.where(z > 0, z, 1)) @ vs, 0.0)
                lse_b = np.where(z[..., 0] > 0, (m + np.log(np.where(z > 0, z, 1)))[..., 0], -np.inf)
            else:
                o_b, lse_b = attention_ref(qs, ks, vs, scale, causal)
            out[q0:q1] = o_b.transpose(1, 0, 2)
            lse[:, q0:q1] = lse_b if kind != "lse_wrong_head" else lse_b[::-1]
        return out, lse
    return fn


@pytest.mark.parametrize("kind", ["query_offsets_for_keys", "one_row_short", "top_left_causal", "lse_wrong_head"])
def test_planted_packing_mistake_is_caught(kind):
    assert _pins(_mutant(kind)) != []


# ---- the packed backward ---------------------------------------------------------------

def test_varlen_backward_matches_finite_differences():
    """Central differences of the packed forward oracle (an independent route to the gradient)
    on a tiny batch with an empty key sequence and more queries than keys."""
    from oracle import attention_varlen_bwd_ref
    lengths = [(3, 4), (2, 0), (4, 2)]
    q, k, v, cu_q, cu_k = _packed(lengths, 2, 3, seed=21)
    do = np.random.default_rng(22).standard_normal(q.shape)
    for causal in (False, True):
        dq, dk, dv = attention_varlen_bwd_ref(q, k, v, do, cu_q, cu_k, 0.6, causal)
        loss = lambda q_, k_, v_: float((attention_varlen_ref(q_, k_, v_, cu_q, cu_k, 0.6, causal)[0] * do).sum())
        eps = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += eps
                xm[idx] -= eps
                args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
                args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
                num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert np.allclose(g, num, atol=1e-6, rtol=1e-5), (name, causal)


def test_varlen_backward_equal_lengths_is_the_batched_oracle():
    from oracle import attention_bwd_ref, attention_varlen_bwd_ref
    B, H, N, d = 3, 2, 6, 4
    rng = np.random.default_rng(23)
    qb, kb, vb, dob = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    pack = lambda x: x.transpose(0, 2, 1, 3).reshape(B * N, H, d)
    cu = np.arange(B + 1) * N
    for causal in (False, True):
        got = attention_varlen_bwd_ref(pack(qb), pack(kb), pack(vb), pack(dob), cu, cu, 0.5, causal)
        ref = attention_bwd_ref(qb, kb, vb, dob, 0.5, causal)
        for a, r in zip(got, ref):
            assert np.allclose(a, pack(r), atol=1e-12, rtol=0)
