"""The forward kernels' work lists (attn_fwd_schedule, host only): every unit exactly once, lists
balanced under the cost of K/V blocks per unit, longest first within a group of heads, and the
first units of all CTAs inside the first group (so that the K and V they stream share the L2)."""

import math

import pytest

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ea_build.build()
    ea.lib()


def _tiles(d):
    return 1 if d == 256 else 2


def _blocks(t, Nq, Nk, causal):
    """K/V blocks of Q tile t: all of them, or, causal, those up to the tile's last row shifted
    by Nk - Nq (bottom-right alignment)."""
    nb, nbk = math.ceil(Nq / 128), math.ceil(Nk / 128)
    if t >= nb:
        return 0
    if not causal:
        return nbk
    last = min(t * 128 + 127, Nq - 1) + Nk - Nq
    return 0 if last < 0 else min(last // 128 + 1, nbk)


def _unit(u, B, H, Nq, d, causal):
    BH = B * H
    T = _tiles(d)
    n_pairs = math.ceil(math.ceil(Nq / 128) / T)
    r = u // BH
    pair = n_pairs - 1 - r if causal else r
    return u % BH, pair * T


def _cost(u, B, H, Nq, Nk, d, causal):
    _, t0 = _unit(u, B, H, Nq, d, causal)
    return max(_blocks(t0 + q, Nq, Nk, causal) for q in range(_tiles(d))) + 2


SHAPES = [(2, 16, 8192, 8192, 128, True), (2, 16, 8192, 8192, 128, False), (1, 32, 16384, 16384, 64, True),
          (2, 8, 8192, 8192, 256, True), (4, 16, 2048, 2048, 128, True), (1, 3, 1000, 1000, 128, True),
          (2, 5, 300, 700, 64, True), (3, 4, 700, 300, 128, True), (1, 1, 129, 129, 256, False),
          (16, 16, 512, 512, 64, False), (1, 64, 16384, 16384, 128, True)]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal", SHAPES)
@pytest.mark.parametrize("num_ctas", [148, 7])
def test_every_unit_once_and_balanced(B, H, Nq, Nk, d, causal, num_ctas):
    lists = ea.attn_fwd_schedule(B, H, Nq, Nk, d, causal=causal, num_ctas=num_ctas)
    n_units = B * H * math.ceil(math.ceil(Nq / 128) / _tiles(d))
    assert len(lists) == min(num_ctas, n_units)
    assert sorted(u for l in lists for u in l) == list(range(n_units))
    loads = [sum(_cost(u, B, H, Nq, Nk, d, causal) for u in l) for l in lists]
    total = sum(loads)
    biggest = max(_cost(u, B, H, Nq, Nk, d, causal) for u in range(n_units))
    # greedy list scheduling: no list exceeds the mean by more than the largest unit
    assert max(loads) <= total / len(lists) + biggest


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal", [s for s in SHAPES if s[5]])
def test_causal_lists_run_longest_first_within_a_group(B, H, Nq, Nk, d, causal):
    lists = ea.attn_fwd_schedule(B, H, Nq, Nk, d, causal=causal)
    # inside one CTA's list the units of one group of heads come longest first
    for l in lists:
        costs = [_cost(u, B, H, Nq, Nk, d, causal) for u in l]
        groups = _group_of(l, B, H, Nq, Nk, d)
        for i in range(len(l) - 1):
            if groups[i] == groups[i + 1]:
                assert costs[i] >= costs[i + 1], (l, costs)


def _group_size(B, H, Nq, Nk, d, elem=2, num_ctas=148):
    BH = B * H
    P = math.ceil(math.ceil(Nq / 128) / _tiles(d))
    g = min(num_ctas, BH * P)
    kv = 2 * Nk * d * elem
    G = min(BH, max(max(1, (32 << 20) // kv), math.ceil(2 * g / P)))
    n_groups = math.ceil(BH / G)
    return math.ceil(BH / n_groups)


def _group_of(l, B, H, Nq, Nk, d):
    G = _group_size(B, H, Nq, Nk, d)
    return [(u % (B * H)) // G for u in l]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal", SHAPES)
def test_first_units_share_one_group_of_heads(B, H, Nq, Nk, d, causal):
    """Every CTA's first unit lies in the first group of heads when that group has at least as
    many units as there are CTAs; the group's K and V fit 32 MB unless fewer heads would leave
    fewer than two units per CTA."""
    lists = ea.attn_fwd_schedule(B, H, Nq, Nk, d, causal=causal)
    BH = B * H
    P = math.ceil(math.ceil(Nq / 128) / _tiles(d))
    G = _group_size(B, H, Nq, Nk, d)
    if G * P >= len(lists):
        assert {l[0] % BH for l in lists} <= set(range(G))
    if 2 * Nk * d * 2 * G > (32 << 20):
        assert G * P <= 2 * len(lists) + P or G == 1


def test_fp8_groups_count_one_byte_elements():
    a = ea.attn_fwd_schedule(2, 16, 8192, 8192, 128, causal=False)
    b = ea.attn_fwd_schedule(2, 16, 8192, 8192, 128, causal=False, fp8=True)
    heads = lambda s: len({l[0] % 32 for l in s})
    assert heads(b) >= heads(a)


def test_huge_launch_keeps_round_robin_and_bad_arguments():
    assert ea.attn_fwd_schedule(1, 1, (1 << 28) + 256, 128, 128) is None
    with pytest.raises(RuntimeError):
        ea.attn_fwd_schedule(1, 1, 128, 128, 96)
    with pytest.raises(RuntimeError):
        ea.attn_fwd_schedule(0, 1, 128, 128, 128)
    with pytest.raises(RuntimeError):
        ea.attn_fwd_schedule(1, 1, 128, 128, 96, fp8=True)
