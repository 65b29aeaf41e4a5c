"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no attention, transform or quantisation arithmetic: it only draws random
numbers and rounds them to the storage type (bf16, round to nearest even).

Recipe (the same for every workload):

* ``numpy.random.default_rng(seed)`` (seed 0 unless stated) draws ``standard_normal``
  float32 arrays for Q, then K, then V, each of shape ``[B, H, N, d]``.
* Outlier workloads then visit Q, K, V in that order: ``mask = rng.random(shape) < frac``
  and the masked entries are replaced by ``rng.normal(0, outlier_std, mask.sum())``.
* Every tensor is rounded to bf16 (round to nearest even) last.
* The random-sign diagonal of the Hadamard transform is ``2 * (default_rng(seed).random(d)
  < 0.5) - 1`` with seed 1, stored as int8 +-1.
* Workloads whose keys differ in length from the queries draw Q ``[B, H, Nq, d]``, then K and
  V ``[B, H, Nk, d]``, in that order, from the same generator.
* The upstream gradient dO of the backward workloads is ``default_rng(seed).standard_normal``
  float32 of shape ``[B, H, N, d]`` with seed 7 unless stated, rounded to bf16.
* Rotary tables: ``cos``/``sin`` ``[n_pos, d/2]`` of the angles ``n * 10000^(-2i/d)``, computed
  in float64 and rounded to float32 once (an input, like the signs: the kernels take any table).
* Packed variable-length workloads: sequence lengths are ``default_rng(seed).integers(lo,
  hi + 1, B)`` (queries; keys the same unless given), the offsets their running sums from 0,
  and Q ``[total_q, H, d]``, K, V ``[total_k, H, d]`` are drawn iid N(0, 1) in that order from
  ``default_rng(seed + 1)``, rounded to bf16.
"""

from __future__ import annotations

import numpy as np


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 array whose values are ``x`` rounded to bfloat16 (ties to even)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    r = ((u + bias) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32)


def bf16_bits(x_bf16_values: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exact bf16 numbers."""
    u = np.ascontiguousarray(x_bf16_values, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def normal_qkv(B: int, H: int, N: int, d: int, seed: int = 0,
               outlier_frac: float = 0.0, outlier_std: float = 10.0):
    """(q, k, v): float32 arrays of bf16 values, shape [B, H, N, d], iid N(0, 1).

    With ``outlier_frac > 0`` that fraction of entries (in expectation) of each tensor is
    replaced by N(0, outlier_std^2) draws before rounding.
    """
    rng = np.random.default_rng(seed)
    shape = (B, H, N, d)
    ts = [rng.standard_normal(shape, dtype=np.float32) for _ in range(3)]
    if outlier_frac > 0.0:
        for t in ts:
            mask = rng.random(shape) < outlier_frac
            t[mask] = rng.normal(0.0, outlier_std, int(mask.sum())).astype(np.float32)
    return tuple(round_to_bf16(t) for t in ts)


def hadamard_signs(d: int, seed: int = 1) -> np.ndarray:
    """int8 vector of +-1 of length d (the random-sign diagonal D)."""
    rng = np.random.default_rng(seed)
    return (2 * (rng.random(d) < 0.5).astype(np.int8) - 1).astype(np.int8)


def normal_dout(B: int, H: int, N: int, d: int, seed: int = 7) -> np.ndarray:
    """dO for the backward workloads: float32 array of bf16 values, [B, H, N, d], iid N(0, 1)."""
    rng = np.random.default_rng(seed)
    return round_to_bf16(rng.standard_normal((B, H, N, d), dtype=np.float32))


def normal_qkv_lengths(B: int, H: int, Nq: int, Nk: int, d: int, seed: int = 0):
    """(q, k, v) with q [B, H, Nq, d] and k, v [B, H, Nk, d]: float32 arrays of bf16 values,
    iid N(0, 1), drawn in the order Q, K, V."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, Nq, d), dtype=np.float32)
    k = rng.standard_normal((B, H, Nk, d), dtype=np.float32)
    v = rng.standard_normal((B, H, Nk, d), dtype=np.float32)
    return round_to_bf16(q), round_to_bf16(k), round_to_bf16(v)


def uniform_lengths(B: int, lo: int, hi: int, seed: int = 0) -> np.ndarray:
    """B sequence lengths drawn uniformly from [lo, hi] (int64)."""
    return np.random.default_rng(seed).integers(lo, hi + 1, B).astype(np.int64)


def normal_qkv_packed(lengths_q, lengths_k, H: int, d: int, seed: int = 0):
    """(q, k, v, cu_q, cu_k) for a packed batch: q [sum(lengths_q), H, d], k, v
    [sum(lengths_k), H, d] float32 arrays of bf16 values, iid N(0, 1), drawn in the order Q, K,
    V; cu_q, cu_k the int32 offsets (B + 1 entries, starting at 0)."""
    cu_q = np.concatenate([[0], np.cumsum(lengths_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lengths_k)]).astype(np.int32)
    rng = np.random.default_rng(seed + 1)
    q = rng.standard_normal((int(cu_q[-1]), H, d), dtype=np.float32)
    k = rng.standard_normal((int(cu_k[-1]), H, d), dtype=np.float32)
    v = rng.standard_normal((int(cu_k[-1]), H, d), dtype=np.float32)
    return round_to_bf16(q), round_to_bf16(k), round_to_bf16(v), cu_q, cu_k


def rope_tables(n_pos: int, d: int, base: float = 10000.0):
    """float32 ``(cos, sin)`` tables ``[n_pos, d/2]`` for the angles ``n * base^(-2i/d)``,
    computed in float64 and rounded once."""
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    ang = np.arange(n_pos, dtype=np.float64)[:, None] * theta[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
