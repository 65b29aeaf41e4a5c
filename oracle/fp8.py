"""FP8 pre-processing oracle (TEST INFRASTRUCTURE ONLY; see ``oracle/__init__.py``).

Follows "FlashAttention-3", section "FP8 路径与低精度误差" ("Incoherent processing 在做什么":
``x~ = H D x`` with ``D`` a diagonal of random signs and ``H`` a Hadamard transform; "为什么
Hadamard 适合放到内核里": an O(d log d) transform) and "FlashAttention-2/3", section
"FA-3：拥抱 Hopper", feature 2 (E4M3/E5M2 formats) and feature 3 (per-block scales).

Readings taken where the pages are silent:

* ``H`` is the Sylvester Hadamard matrix of order d, normalised by ``1/sqrt(d)`` so that
  ``H D`` is orthogonal and ``(HDq).(HDk) = q.k``: scores do not change.
* One sign vector of length d serves every head and both Q and K; V is quantised without
  the transform.
* E4M3 is the OCP E4M3FN format (bias 7, max 448, no infinities), rounding to nearest
  even, saturating at +-448.
* A block is 128 consecutive rows of one (batch, head).  With ``y = H_d (D x)`` the
  unnormalised transform, the block's unit scale is ``s_u = max(amax(|y|) / 448, 2^-126)``
  and the stored code is ``e4m3(y * (1 / s_u))``; the stored scale is
  ``s = s_u * (1/sqrt(d))`` so that ``code * s`` approximates ``x~`` (for V: ``s = s_u``).
  Normalising after the quantisation decision gives the same codes as normalising first
  in exact arithmetic and keeps the irrational ``1/sqrt(d)`` out of the decision.
* The quantisation decision is an integer chosen by floating point, so it is taken in the
  precision the kernel takes it in: the transform is the textbook butterfly (stages of
  stride 1, 2, 4, ...) in float32, and ``amax / 448``, ``1 / s_u``, ``y * (1/s_u)`` and
  ``s_u * (1/sqrt(d))`` are single IEEE float32 operations.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUBNORMAL_QUANTUM = 2.0 ** -9
QUANT_BLOCK = 128
F32_MIN_NORMAL = np.float32(2.0 ** -126)


def sylvester_hadamard(d: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix: H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_rotate_ref(x, signs) -> np.ndarray:
    """x~ = (1/sqrt(d)) H_d D x for every row of ``x`` (float64, explicit matrix product)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = sylvester_hadamard(d)
    return (x * np.asarray(signs, dtype=np.float64)) @ h.T / np.sqrt(d)


def fwht_f32(y) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform of each row, in float32.

    log2(d) butterfly stages of stride h = 1, 2, 4, ..., d/2: the pair (a, b) at positions
    (i, i + h) inside each group of 2h becomes (a + b, a - b).  Equals ``H_d @ y`` in exact
    arithmetic; every add and subtract is one float32 rounding.
    """
    y = np.array(y, dtype=np.float32, copy=True)
    d = y.shape[-1]
    lead = y.shape[:-1]
    h = 1
    while h < d:
        t = y.reshape(lead + (d // (2 * h), 2, h))
        a = t[..., 0, :]
        b = t[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2).reshape(lead + (d,))
        h *= 2
    return y


def e4m3_round(x) -> np.ndarray:
    """Round float64 values to the nearest E4M3FN value (ties to even), saturating at +-448.

    Normal range: |x| in [2^-6, 448] with 3 fraction bits, so the spacing at exponent e is
    2^(e-3).  Below 2^-6 the spacing is the subnormal quantum 2^-9.  Scaling by powers of
    two and ``np.rint`` (ties to even) are exact in float64.  NaN stays NaN.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))  # a = m * 2**ex, m in [0.5, 1)
    e = ex - 1  # floor(log2 a)
    quantum = np.where(a < E4M3_MIN_NORMAL, E4M3_SUBNORMAL_QUANTUM, np.ldexp(1.0, e - 3))
    r = np.rint(a / quantum) * quantum
    r = np.minimum(r, E4M3_MAX)
    r = np.where(np.isnan(x), np.nan, r)
    return np.copysign(r, x)


def e4m3_encode(values) -> np.ndarray:
    """Bit patterns (uint8) of values that are already exact E4M3FN numbers."""
    v = np.asarray(values, dtype=np.float64)
    sign = np.signbit(v).astype(np.uint8) << 7
    a = np.abs(v)
    code = np.zeros(v.shape, dtype=np.uint8)
    sub = (a < E4M3_MIN_NORMAL)
    code = np.where(sub, np.rint(a / E4M3_SUBNORMAL_QUANTUM), code)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = ex - 1
    frac = np.rint((a / np.ldexp(1.0, e) - 1.0) * 8.0)
    normal = (e + 7) * 8 + frac
    code = np.where(sub, code, normal)
    code = np.where(np.isnan(v), 0x7F, code).astype(np.uint8)
    return code | sign


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of E4M3FN bit patterns (0x7F / 0xFF are NaN)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * E4M3_SUBNORMAL_QUANTUM, np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return s * val


def hadamard_quant_ref(x, signs=None, block: int = QUANT_BLOCK):
    """Per-block E4M3 quantisation of ``x`` ([..., N, d], bf16 values as float64).

    With ``signs`` (length d, entries +-1) the rows are first transformed,
    ``y = H_d (D x)`` in float32 (``fwht_f32``); without, ``y = x``.  For every block of
    ``block`` rows of one leading index: ``s_u = max(amax/448, 2^-126)``, codes
    ``e4m3(y * (1/s_u))``, stored scale ``s_u * (1/sqrt(d))`` (Hadamard) or ``s_u``.

    Returns ``(codes uint8 [..., N, d], scales float32 [..., ceil(N/block)])``.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    n = x.shape[-2]
    lead = x.shape[:-2]
    y = x.astype(np.float32)
    if signs is not None:
        y = fwht_f32(y * np.asarray(signs, dtype=np.float32))
        post = np.float32(1.0 / np.sqrt(d))
    else:
        post = np.float32(1.0)
    y3 = y.reshape((-1, n, d))
    nb = (n + block - 1) // block
    codes = np.zeros(y3.shape, dtype=np.uint8)
    scales = np.zeros((y3.shape[0], nb), dtype=np.float32)
    for g in range(y3.shape[0]):
        for blk in range(nb):
            r0, r1 = blk * block, min(n, (blk + 1) * block)
            yb = y3[g, r0:r1]
            amax = np.float32(np.abs(yb).max())
            s_u = np.float32(amax / np.float32(E4M3_MAX))
            s_u = max(s_u, F32_MIN_NORMAL)
            r = np.float32(np.float32(1.0) / s_u)
            q = (yb * r).astype(np.float32)  # one float32 multiply per element
            codes[g, r0:r1] = e4m3_encode(e4m3_round(q.astype(np.float64)))
            scales[g, blk] = np.float32(s_u * post)
    return codes.reshape(lead + (n, d)), scales.reshape(lead + (nb,))


def dequant_ref(codes, scales, block: int = QUANT_BLOCK) -> np.ndarray:
    """float64 ``code * scale`` with one scale per block of ``block`` rows."""
    vals = e4m3_decode(codes)
    n = vals.shape[-2]
    rep = np.repeat(np.asarray(scales, dtype=np.float64), block, axis=-1)[..., :n]
    return vals * rep[..., None]
