"""Fits the cubic used by the kernels' FMA-pipe exp2 and prints its float32 coefficients.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is replaced by
c0 + c1 f + c2 f^2 + c3 f^3.  The coefficients minimise the maximum relative error on
[-1/2, 1/2]: a relative-error least-squares fit at Chebyshev nodes, refined by iteratively
reweighting toward the error extrema (Lawson's algorithm), in float64, then rounded to
float32.  Run with no arguments; the printed values are the ones in csrc/attn_fwd_kernel.cuh.
"""

import numpy as np


def fit(degree: int = 3, nodes: int = 2001, iters: int = 200):
    t = np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes) * 0.5  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(t)
    A = np.vander(t, degree + 1, increasing=True) / y[:, None]  # relative error: (p - y) / y
    b = np.ones_like(t)
    w = np.ones_like(t) / nodes
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def max_rel_error_f32(c):
    """Max relative error of the float32 evaluation (Horner) against 2^f, on a dense grid."""
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.float32(c[3])
    for k in (2, 1, 0):
        p = (p * f + np.float32(c[k])).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for k, v in enumerate(c):
        print(f"c{k} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print("max relative error (float32 Horner):", max_rel_error_f32(c))
