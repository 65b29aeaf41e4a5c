"""Rotary position embedding oracle (TEST INFRASTRUCTURE ONLY; see ``oracle/__init__.py``).

"FlashAttention-3", section "为什么 Hadamard 适合放到内核里": the Hadamard transform is
memory-bound and can be fused with RoPE, another bandwidth-bound pre-processing step.  The
pages name RoPE but do not define it; the reading taken is the usual rotary embedding in its
rotate-half pairing: coordinate i and coordinate i + d/2 of a row form a plane, rotated by the
angle that the caller's tables give for the row's position:

    y_i       = x_i       * cos[n, i] - x_{i+d/2} * sin[n, i]
    y_{i+d/2} = x_{i+d/2} * cos[n, i] + x_i       * sin[n, i]        (0 <= i < d/2)

for row n of each sequence, with ``cos`` and ``sin`` tables of shape ``[n_pos, d/2]``
(``n_pos >= N``) that the caller fills (e.g. ``cos(n * base^(-2i/d))``).  Fused with the FP8
pre-processing, the rotated rows then go through ``x~ = H D x`` and the per-block E4M3
quantisation of ``oracle.fp8``.  Because those codes are integers chosen by floating point,
the rotation is taken in the kernel's precision: float32, each product rounded, then the
difference or sum rounded (no fused multiply-add).
"""

from __future__ import annotations

import numpy as np


def rope_ref(x, cos, sin) -> np.ndarray:
    """Rotate-half rotary embedding of every row of ``x`` ([..., N, d]) in float32.

    Row n takes ``cos[n]`` and ``sin[n]`` (tables ``[n_pos, d/2]``, ``n_pos >= N``).
    Returns float32 ``[..., N, d]``.
    """
    x = np.asarray(x, dtype=np.float32)
    n, d = x.shape[-2], x.shape[-1]
    half = d // 2
    c = np.asarray(cos, dtype=np.float32)[:n]
    s = np.asarray(sin, dtype=np.float32)[:n]
    a = x[..., :half]
    b = x[..., half:]
    # numpy float32 arithmetic rounds every operation: products first, then the sum
    y_lo = (a * c).astype(np.float32) - (b * s).astype(np.float32)
    y_hi = (b * c).astype(np.float32) + (a * s).astype(np.float32)
    return np.concatenate([y_lo.astype(np.float32), y_hi.astype(np.float32)], axis=-1)

