"""float64 oracle of the attention backward pass (TEST INFRASTRUCTURE ONLY; see ``oracle/__init__.py``).

The pages state that the backward pass exists for FP16/BF16 ("FlashAttention-3", section
"适用范围和工程限制"), that it recomputes the softmax instead of storing it ("Flash
Attention V3 解析", section 2.1, "反向重计算"), and that dQ is accumulated across K/V blocks
(section 4.2, "dQ更新时").  They do not write the gradient out; it is the chain rule applied
to the forward definition, which is what this module evaluates, on whole score matrices:

    S = scale * Q K^T          P = softmax(S) over the visible keys of each row
    O = P V
    dV = P^T dO                dP = dO V^T
    dS = P * (dP - rowsum(P * dP))            (the softmax Jacobian applied row by row)
    dQ = scale * dS K          dK = scale * dS^T Q

``rowsum(P * dP)`` equals ``rowsum(dO * O)`` (both are sum_j P_ij sum_c dO_ic V_jc); the
second form is the one a tiled kernel can compute before its loops, from O alone.

All arrays are float64 ``[..., N, d]``; leading dimensions are independent problems.
"""

from __future__ import annotations

import numpy as np

from .attention import visible_mask


def _as_3d(x: np.ndarray):
    lead = x.shape[:-2]
    return x.reshape((-1,) + x.shape[-2:]), lead


def softmax_probs(q, k, scale: float, causal: bool = False) -> np.ndarray:
    """P = softmax(scale * Q K^T) over the visible keys, float64 ``[..., N_q, N_k]``."""
    q3, lead = _as_3d(np.asarray(q, dtype=np.float64))
    k3, _ = _as_3d(np.asarray(k, dtype=np.float64))
    s = scale * np.einsum("bid,bjd->bij", q3, k3)
    vis = visible_mask(q3.shape[1], k3.shape[1], causal)
    s = np.where(vis[None], s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(vis[None], np.exp(s - m), 0.0)
    den = e.sum(axis=-1, keepdims=True)
    p = np.divide(e, den, out=np.zeros_like(e), where=den > 0)
    return p.reshape(lead + p.shape[-2:])


def softmax_bwd_delta(o, do) -> np.ndarray:
    """D_i = sum_c dO_ic O_ic, float64 ``[..., N]`` (equal to rowsum(P * dP))."""
    return np.einsum("...ic,...ic->...i", np.asarray(do, dtype=np.float64), np.asarray(o, dtype=np.float64))


def attention_bwd_ref(q, k, v, do, scale: float, causal: bool = False):
    """(dQ, dK, dV) of ``O = softmax(scale Q K^T) V`` for the upstream gradient ``dO``, float64.

    Straight from the definition above: P is formed in full, dS uses rowsum(P * dP).
    """
    q3, lead = _as_3d(np.asarray(q, dtype=np.float64))
    k3, _ = _as_3d(np.asarray(k, dtype=np.float64))
    v3, _ = _as_3d(np.asarray(v, dtype=np.float64))
    do3, _ = _as_3d(np.asarray(do, dtype=np.float64))
    p = softmax_probs(q3, k3, scale, causal)
    dv = np.einsum("bij,bic->bjc", p, do3)
    dp = np.einsum("bic,bjc->bij", do3, v3)
    ds = p * (dp - (p * dp).sum(axis=-1, keepdims=True))
    dq = scale * np.einsum("bij,bjc->bic", ds, k3)
    dk = scale * np.einsum("bij,bic->bjc", ds, q3)
    return dq.reshape(q.shape), dk.reshape(k.shape), dv.reshape(v.shape)


def attention_bwd_chunked_ref(q, k, v, do, scale: float, causal: bool = False, row_chunk: int = 1024):
    """(dQ, dK, dV) of :func:`attention_bwd_ref`, evaluated ``row_chunk`` query rows at a time.

    The same chain rule on the same definition, for problems whose full score matrix does not
    fit in memory (N = 8192 and beyond).  For every block of query rows ``c`` it forms
    ``P_c`` (softmax over the visible keys of those rows), ``dP_c = dO_c V^T`` and
    ``dS_c = P_c * (dP_c - rowsum(P_c * dP_c))``; ``dQ_c = scale dS_c K`` is complete within the
    block, while ``dV = sum_c P_c^T dO_c`` and ``dK = scale sum_c dS_c^T Q_c`` are summed over the
    blocks.  Only the order of the float64 sums differs from the whole-matrix form.  Inputs are
    ``[..., N, d]`` (``k``, ``v`` may have another length than ``q``; causal masking is
    bottom-right aligned as in :func:`oracle.attention.visible_mask`).
    """
    q3, _ = _as_3d(np.asarray(q, dtype=np.float64))
    k3, _ = _as_3d(np.asarray(k, dtype=np.float64))
    v3, _ = _as_3d(np.asarray(v, dtype=np.float64))
    do3, _ = _as_3d(np.asarray(do, dtype=np.float64))
    g, n_q, _ = q3.shape
    n_k = k3.shape[1]
    dq, dk, dv = np.zeros_like(q3), np.zeros_like(k3), np.zeros_like(v3)
    for b in range(g):
        for r0 in range(0, n_q, row_chunk):
            r1 = min(n_q, r0 + row_chunk)
            s = scale * (q3[b, r0:r1] @ k3[b].T)
            vis = visible_mask(n_q, n_k, causal)[r0:r1]
            s = np.where(vis, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            e = np.where(vis, np.exp(s - m), 0.0)
            den = e.sum(axis=1, keepdims=True)
            p = np.divide(e, den, out=np.zeros_like(e), where=den > 0)
            dv[b] += p.T @ do3[b, r0:r1]
            dp = do3[b, r0:r1] @ v3[b].T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dq[b, r0:r1] = scale * (ds @ k3[b])
            dk[b] += scale * (ds.T @ q3[b, r0:r1])
    return dq.reshape(np.shape(q)), dk.reshape(np.shape(k)), dv.reshape(np.shape(v))


def attention_varlen_bwd_ref(q, k, v, do, cu_q, cu_k, scale: float, causal: bool = False):
    """(dQ, dK, dV) of the packed batch ``attention_varlen_ref`` defines, float64.

    ``q``, ``do`` are ``[total_q, H, d]``, ``k``, ``v`` ``[total_k, H, d]``; sequence ``b`` owns
    query rows ``cu_q[b]:cu_q[b+1]`` and key rows ``cu_k[b]:cu_k[b+1]``.  Each sequence is its
    own problem, so its gradients are :func:`attention_bwd_ref` of its own rows; a sequence with
    no keys (or no queries) has zero gradients, and rows outside every sequence stay zero.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0 or k1 == k0:
            continue
        t = lambda x: x.transpose(1, 0, 2)  # [rows, H, d] <-> [H, rows, d]
        g = attention_bwd_ref(t(q[q0:q1]), t(k[k0:k1]), t(v[k0:k1]), t(do[q0:q1]), scale, causal)
        dq[q0:q1], dk[k0:k1], dv[k0:k1] = (t(x) for x in g)
    return dq, dk, dv
