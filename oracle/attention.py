"""float64 attention oracle (TEST INFRASTRUCTURE ONLY; see ``oracle/__init__.py``).

Three independent computations of the same result:

``attention_ref``                 the definition, two passes per row block (max, then exp/sum).
``attention_blockwise_ref``       the tiled recurrence exactly as "FlashAttention-2/3",
                                  section "技术原理", states it (outer loop over Q blocks, inner
                                  loop over K/V blocks, running m and l, O corrected each step).
``attention_blockwise_lazy_ref``  the same recurrence in base 2 with the normalisation moved
                                  to the end ("FlashAttention-2/3", FA-2 improvement 1;
                                  "Flash Attention V3 解析" section 2.2) and the reference max
                                  updated only when it grows by more than ``tau``.

All arrays are float64 with shape ``[..., N, d]``; leading dimensions (batch, heads) are
independent problems.  Scores are ``s_ij = scale * q_i . k_j``; the caller passes
``scale`` (the pages' formula uses ``1/sqrt(d)``).
"""

from __future__ import annotations

import numpy as np

LOG2E = 1.4426950408889634  # log2(e)
LN2 = 0.6931471805599453  # ln(2)


def visible_mask(n_q: int, n_k: int, causal: bool) -> np.ndarray:
    """Boolean ``[n_q, n_k]``: key j is visible to query i.

    The pages do not state how a causal mask aligns when the query and key lengths differ;
    the reading taken is bottom-right alignment, ``j <= i + (n_k - n_q)``, which is the
    plain ``j <= i`` whenever the lengths are equal.
    """
    if not causal:
        return np.ones((n_q, n_k), dtype=bool)
    i = np.arange(n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return j <= i + (n_k - n_q)


def _as_3d(x: np.ndarray) -> tuple[np.ndarray, tuple]:
    lead = x.shape[:-2]
    return x.reshape((-1,) + x.shape[-2:]), lead


def attention_ref(q, k, v, scale: float, causal: bool = False, row_chunk: int = 1024):
    """O = softmax(scale * Q K^T) V and LSE_i = log sum_j exp(s_ij), in float64.

    The definition ("FlashAttention-3", intro formula; "FlashAttention-2/3", "技术原理",
    standard attention steps 1-3), evaluated a block of ``row_chunk`` query rows at a time
    so that memory stays bounded; each block takes the row max first and then the
    exponentials, sum and weighted sum (two passes over the scores).

    Returns ``(O, LSE)`` with shapes ``[..., N_q, d_v]`` and ``[..., N_q]``.  A row with no
    visible key (impossible when ``N_q == N_k``) gets ``O = 0`` and ``LSE = -inf``.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    q3, lead = _as_3d(q)
    k3, _ = _as_3d(k)
    v3, _ = _as_3d(v)
    g, n_q, _ = q3.shape
    n_k = k3.shape[1]
    d_v = v3.shape[2]
    out = np.zeros((g, n_q, d_v), dtype=np.float64)
    lse = np.full((g, n_q), -np.inf, dtype=np.float64)
    for b in range(g):
        for r0 in range(0, n_q, row_chunk):
            r1 = min(n_q, r0 + row_chunk)
            s = scale * (q3[b, r0:r1] @ k3[b].T)  # [rows, n_k]
            if causal:
                vis = visible_mask(n_q, n_k, True)[r0:r1]
                s = np.where(vis, s, -np.inf)
            m = s.max(axis=1)  # pass 1: row max
            has = np.isfinite(m)
            m_safe = np.where(has, m, 0.0)
            e = np.exp(s - m_safe[:, None])  # pass 2: exponentials (exp(-inf) = 0)
            l = e.sum(axis=1)
            with np.errstate(divide="ignore", invalid="ignore"):
                p = np.where(has[:, None], e / np.where(has, l, 1.0)[:, None], 0.0)
                lse[b, r0:r1] = np.where(has, m_safe + np.log(np.where(has, l, 1.0)), -np.inf)
            out[b, r0:r1] = p @ v3[b]
    return out.reshape(lead + (n_q, d_v)), lse.reshape(lead + (n_q,))


def attention_blockwise_ref(q, k, v, scale: float, causal: bool, block_r: int, block_c: int):
    """The tiled recurrence of "FlashAttention-2/3", section "技术原理", in float64.

    Q is cut into blocks of ``block_r`` rows (the pages' B_r, T_r blocks), K and V into
    blocks of ``block_c`` rows (B_c, T_c blocks).  For each Q block, with ``O_i = 0,
    l_i = 0, m_i = -inf``, every K/V block does, in the pages' order:

        S_ij = Q_i K_j^T (times ``scale``; the pseudocode leaves the 1/sqrt(d) implicit)
        m_ij = rowmax(S_ij);  P_ij = exp(S_ij - m_ij);  l_ij = rowsum(P_ij)
        m_new = max(m_i, m_ij)
        l_new = l_i exp(m_i - m_new) + l_ij exp(m_ij - m_new)
        O_i   = O_i (l_i exp(m_i - m_new) / l_new) + (exp(m_ij - m_new) / l_new) P_ij V_j
        m_i, l_i = m_new, l_new

    The pseudocode then divides O_i by l_i once more; since the update above already keeps
    O_i normalised, that final division would normalise twice (a garbled step), so it is
    not applied.  LSE_i = m_i + log l_i.  Masked scores are -inf; a block row with no
    visible key contributes nothing (P = 0, l_ij = 0, exp(m_ij - m_new) taken as 0).
    """
    q3, lead = _as_3d(np.asarray(q, dtype=np.float64))
    k3, _ = _as_3d(np.asarray(k, dtype=np.float64))
    v3, _ = _as_3d(np.asarray(v, dtype=np.float64))
    g, n_q, _ = q3.shape
    n_k = k3.shape[1]
    d_v = v3.shape[2]
    vis_all = visible_mask(n_q, n_k, causal)
    out = np.zeros((g, n_q, d_v))
    lse = np.zeros((g, n_q))
    for b in range(g):
        for r0 in range(0, n_q, block_r):
            r1 = min(n_q, r0 + block_r)
            o_i = np.zeros((r1 - r0, d_v))
            l_i = np.zeros(r1 - r0)
            m_i = np.full(r1 - r0, -np.inf)
            for c0 in range(0, n_k, block_c):
                c1 = min(n_k, c0 + block_c)
                s_ij = scale * (q3[b, r0:r1] @ k3[b, c0:c1].T)
                s_ij = np.where(vis_all[r0:r1, c0:c1], s_ij, -np.inf)
                m_ij = s_ij.max(axis=1)
                any_vis = np.isfinite(m_ij)
                p_ij = np.where(any_vis[:, None], np.exp(s_ij - np.where(any_vis, m_ij, 0.0)[:, None]), 0.0)
                l_ij = p_ij.sum(axis=1)
                m_new = np.maximum(m_i, m_ij)
                live = np.isfinite(m_new)
                m_new_safe = np.where(live, m_new, 0.0)
                a_old = np.where(np.isfinite(m_i), np.exp(m_i - m_new_safe), 0.0)
                a_new = np.where(any_vis, np.exp(np.where(any_vis, m_ij, 0.0) - m_new_safe), 0.0)
                l_new = l_i * a_old + l_ij * a_new
                with np.errstate(divide="ignore", invalid="ignore"):
                    inv = np.where(l_new > 0, 1.0 / np.where(l_new > 0, l_new, 1.0), 0.0)
                o_i = o_i * (l_i * a_old * inv)[:, None] + (a_new * inv)[:, None] * (p_ij @ v3[b, c0:c1])
                m_i, l_i = m_new, l_new
            out[b, r0:r1] = o_i
            with np.errstate(divide="ignore"):
                lse[b, r0:r1] = np.where(l_i > 0, m_i + np.log(np.where(l_i > 0, l_i, 1.0)), -np.inf)
    return out.reshape(lead + (n_q, d_v)), lse.reshape(lead + (n_q,))


def attention_blockwise_lazy_ref(q, k, v, scale: float, causal: bool, block_c: int, tau: float):
    """Deferred-normalisation recurrence in base 2 with a lazily updated reference max.

    Restates the FA-2 form ("FlashAttention-2/3", FA-2 improvement 1: rescaling moved out
    of the inner loop; "Flash Attention V3 解析" section 2.2: normalise at the end, keep the
    logsumexp) with two rewrites that leave the result unchanged in exact arithmetic:

    * ``exp(s) = 2 ** (s * log2 e)``: scores are taken in base 2, ``x = s * scale * log2 e``;
    * the reference max ``m`` used for ``p = 2 ** (x - m)`` moves to a new block maximum
      only when that maximum exceeds it by more than ``tau``; the unnormalised accumulator
      ``O~`` and the running sum ``l`` are then both multiplied by ``2 ** (m_old - m_new)``.
      Both are always relative to the same ``m``, so ``O = O~ / l`` is exact for any
      ``tau >= 0``, and ``p <= 2 ** tau`` bounds the growth.

    Final ``O = O~ / l`` and ``LSE = (m + log2 l) * ln 2``.  Rows are processed one key block
    of ``block_c`` at a time (all query rows at once; the row tiling does not change the
    per-row arithmetic).
    """
    q3, lead = _as_3d(np.asarray(q, dtype=np.float64))
    k3, _ = _as_3d(np.asarray(k, dtype=np.float64))
    v3, _ = _as_3d(np.asarray(v, dtype=np.float64))
    g, n_q, _ = q3.shape
    n_k = k3.shape[1]
    d_v = v3.shape[2]
    vis_all = visible_mask(n_q, n_k, causal)
    c = scale * LOG2E
    out = np.zeros((g, n_q, d_v))
    lse = np.zeros((g, n_q))
    for b in range(g):
        o_acc = np.zeros((n_q, d_v))
        l = np.zeros(n_q)
        m = np.full(n_q, -np.inf)
        for c0 in range(0, n_k, block_c):
            c1 = min(n_k, c0 + block_c)
            x = c * (q3[b] @ k3[b, c0:c1].T)
            x = np.where(vis_all[:, c0:c1], x, -np.inf)
            m_blk = x.max(axis=1)
            with np.errstate(invalid="ignore"):
                grow = np.where(np.isfinite(m), m_blk - m > tau, np.isfinite(m_blk))
            m_new = np.where(grow, m_blk, m)
            alpha = np.where(grow, np.where(np.isfinite(m), np.exp2(m - np.where(grow, m_new, 0.0)), 0.0), 1.0)
            o_acc *= alpha[:, None]
            l *= alpha
            m = m_new
            live = np.isfinite(m)
            p = np.where(live[:, None], np.exp2(x - np.where(live, m, 0.0)[:, None]), 0.0)
            l += p.sum(axis=1)
            o_acc += p @ v3[b, c0:c1]
        with np.errstate(divide="ignore", invalid="ignore"):
            out[b] = np.where((l > 0)[:, None], o_acc / np.where(l > 0, l, 1.0)[:, None], 0.0)
            lse[b] = np.where(l > 0, (m + np.log2(np.where(l > 0, l, 1.0))) * LN2, -np.inf)
    return out.reshape(lead + (n_q, d_v)), lse.reshape(lead + (n_q,))


def attention_varlen_ref(q, k, v, cu_q, cu_k, scale: float, causal: bool = False):
    """A packed batch of independent sequences of different lengths, in float64.

    ``q`` is ``[total_q, H, d]`` and ``k``, ``v`` are ``[total_k, H, d]``; sequence ``b`` owns
    query rows ``cu_q[b]:cu_q[b+1]`` and key/value rows ``cu_k[b]:cu_k[b+1]``.  Each sequence and
    head is the problem :func:`attention_ref` defines (its own causal alignment, from its own
    two lengths); the pages motivate variable context lengths ("FlashAttention-2/3") but fix no
    packing, so this one is the plain reading: rows of one sequence are contiguous.

    Returns ``(O [total_q, H, d_v], LSE [H, total_q])``.  A sequence with no keys gives its
    rows ``O = 0``, ``LSE = -inf``; rows that belong to no sequence stay ``0`` / ``-inf``.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    total_q, h, _ = q.shape
    out = np.zeros((total_q, h, v.shape[2]), dtype=np.float64)
    lse = np.full((h, total_q), -np.inf, dtype=np.float64)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0 or k1 == k0:
            continue  # no rows, or no keys: O = 0, LSE = -inf as initialised
        o_b, lse_b = attention_ref(q[q0:q1].transpose(1, 0, 2), k[k0:k1].transpose(1, 0, 2),
                                   v[k0:k1].transpose(1, 0, 2), scale, causal)
        out[q0:q1] = o_b.transpose(1, 0, 2)
        lse[:, q0:q1] = lse_b
    return out, lse


def merge_partials_ref(o_a, lse_a, o_b, lse_b):
    """Combine two attention results of the same queries over disjoint key sets, float64.

    With ``l = exp(LSE)`` the softmax denominator of each part, the result over the union of the
    keys is ``O = (l_a O_a + l_b O_b) / (l_a + l_b)`` and ``LSE = log(l_a + l_b)``: the running
    rescale of the pages' tiled recurrence ("FlashAttention-2/3", "技术原理") applied to two
    finished parts, and the merge a sequence-sharded (ring) attention needs (the same page names
    long-context parallel systems).  A part with ``LSE = -inf`` (no visible key) contributes
    nothing; if both are ``-inf`` the result is ``O = 0``, ``LSE = -inf``.
    Shapes: O ``[..., N, d]``, LSE ``[..., N]``.
    """
    o_a, o_b = np.asarray(o_a, dtype=np.float64), np.asarray(o_b, dtype=np.float64)
    lse_a, lse_b = np.asarray(lse_a, dtype=np.float64), np.asarray(lse_b, dtype=np.float64)
    m = np.maximum(lse_a, lse_b)
    has = np.isfinite(m)
    m0 = np.where(has, m, 0.0)
    wa = np.where(np.isfinite(lse_a), np.exp(lse_a - m0), 0.0)
    wb = np.where(np.isfinite(lse_b), np.exp(lse_b - m0), 0.0)
    tot = wa + wb
    with np.errstate(divide="ignore", invalid="ignore"):
        o = np.where(has[..., None], (wa[..., None] * o_a + wb[..., None] * o_b) / np.where(has, tot, 1.0)[..., None],
                     0.0)
        lse = np.where(has, m0 + np.log(np.where(has, tot, 1.0)), -np.inf)
    return o, lse
