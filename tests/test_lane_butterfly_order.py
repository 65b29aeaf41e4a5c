"""The order of operations of the d = 256 pre-kernel's lane stages, checked on the CPU.

At d = 256 the pre-kernel spreads a row over four lanes of 64 elements, so the butterflies of
stride 64 and 128 pair elements held by different lanes.  Each lane of a pair keeps half of the
positions, receives the partner's values for those, and computes both outputs of each of its
butterflies as fl(b r + a v) with a, b = +-1 (v its own value, r the received one); the odd
lanes hold the two halves of their part swapped, so that every lane sends the same registers.
This file restates that schedule in float32 numpy -- the lane of each value at each step, the
multipliers, one rounding per output -- and checks that it gives the sequential transform
(``oracle.fwht_f32``) bit for bit, signs of zero included, on rows built to cancel.  The GPU
tests check the kernel itself against the oracle; this one checks the schedule's arithmetic on
any machine."""

import numpy as np
import pytest

from oracle.fp8 import fwht_f32

F32 = np.float32


def _fl(b, r, a, v):
    """fl(b * r + a * v) for b, a = +-1: both products exact, one float32 rounding."""
    return (F32(b) * r + F32(a) * v).astype(F32)


def _four_lane_transform(x, slip=False):
    """x: [rows, 256] float32 (after the sign flips of D).  Returns the transform, as the lanes
    leave it, reassembled in element order.  ``slip``: lane 1 computes its stride-64 differences
    as fl(v - r), its operands reversed (a mistake the check must catch)."""
    rows = x.shape[0]
    lanes = []
    for p in range(4):
        sh = 32 * (p & 1)  # odd lanes: halves of the part swapped
        idx = [64 * p + ((j + sh) & 63) for j in range(64)]
        lanes.append(x[:, idx].copy())
    # strides 1 .. 16 inside each half of a lane's part (natural order within a half)
    for p in range(4):
        v = lanes[p]
        h = 1
        while h < 32:
            for e in range(64):
                if e & h == 0:
                    a, b = v[:, e].copy(), v[:, e + h].copy()
                    v[:, e], v[:, e + h] = (a + b).astype(F32), (a - b).astype(F32)
            h <<= 1
    # stride 32 inside the lane, with the odd lanes' swapped halves
    for p in range(4):
        v = lanes[p]
        s1 = -1.0 if p & 1 else 1.0
        lo, hi = v[:, :32].copy(), v[:, 32:].copy()
        v[:, :32] = _fl(1.0, hi, s1, lo)
        v[:, 32:] = _fl(-s1, hi, 1.0, lo)
    # stride 64 between lanes p and p ^ 1: every lane sends v[32 + t], keeps v[t]
    sent = [lanes[p][:, 32:].copy() for p in range(4)]
    for p in range(4):
        r, v = sent[p ^ 1], lanes[p][:, :32].copy()
        a1, b1 = (-1.0 if p == 3 else 1.0), (-1.0 if p == 2 else 1.0)
        a2, b2 = (-1.0 if p == 1 else 1.0), (-1.0 if p == 0 else 1.0)
        lanes[p][:, :32] = _fl(b1, r, a1, v)
        lanes[p][:, 32:] = (v - r).astype(F32) if (slip and p == 1) else _fl(b2, r, a2, v)
    # stride 128 between lanes p and p ^ 2
    sent = [lanes[p][:, 32:].copy() for p in range(4)]
    for p in range(4):
        r, v = sent[p ^ 2], lanes[p][:, :32].copy()
        a = -1.0 if p >= 2 else 1.0
        lanes[p][:, :32] = (v + r).astype(F32)
        lanes[p][:, 32:] = _fl(-a, r, a, v)
    out = np.empty((rows, 256), dtype=F32)
    for p in range(4):  # lane p ends with elements 32p .. and 128 + 32p ..
        out[:, 32 * p:32 * p + 32] = lanes[p][:, :32]
        out[:, 128 + 32 * p:128 + 32 * p + 32] = lanes[p][:, 32:]
    return out


def _rows(seed):
    rng = np.random.default_rng(seed)
    rows = [
        rng.standard_normal(256),
        np.zeros(256),
        -np.zeros(256),
        rng.choice([0.0, -0.0, 1.0, -1.0, 2.0], 256),
        np.repeat(rng.standard_normal(8), 32),
        rng.integers(-2, 3, 256) * 0.5,
        np.tile([1.5, -1.5], 128),
        np.where(np.arange(256) % 3 == 0, -2.0, 0.0),
    ]
    return np.array(rows, dtype=F32)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_lane_schedule_equals_the_sequential_transform(seed):
    x = _rows(seed)
    signs = np.where(np.random.default_rng(seed + 10).random(256) < 0.5, -1.0, 1.0).astype(F32)
    y = (x * signs).astype(F32)
    got = _four_lane_transform(y)
    want = fwht_f32(y)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_a_plausible_slip_is_caught():
    """Lane 1 computing its stride-64 differences as fl(v - r) instead of fl(r - v) changes the
    result, so the test above would see it."""
    y = _rows(0)
    want = fwht_f32(y)
    assert np.array_equal(_four_lane_transform(y).view(np.uint32), want.view(np.uint32))
    assert not np.array_equal(_four_lane_transform(y, slip=True).view(np.uint32), want.view(np.uint32))
