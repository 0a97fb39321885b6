"""Pins for oracle.allocation: exhaustive brute force on tiny heads, the exact
budget, uniform widths under equal energies, monotonicity, the width cap, and
the energy definition by exact rational arithmetic."""
import itertools
from fractions import Fraction

import numpy as np
import pytest

from oracle import allocation, lloyd_max, rope

DIST = lloyd_max.distortion_table(8)


def _brute_force(e, budget, max_bits=8):
    n = len(e)
    target = budget * n          # sum b_i = budget * d / 2 = budget * n
    best, best_cost = [], None
    for b in itertools.product(range(max_bits + 1), repeat=n):
        if sum(b) != target:
            continue
        cost = sum(float(ei) * DIST[bi] for ei, bi in zip(e, b))
        if best_cost is None or cost < best_cost - 1e-15:
            best, best_cost = [b], cost
        elif abs(cost - best_cost) <= 1e-15:
            best.append(b)
    return best, best_cost


@pytest.mark.parametrize("d", [4, 6, 8, 10])
@pytest.mark.parametrize("budget", [1, 2, 3, 4])
def test_greedy_matches_brute_force(d, budget):
    rng = np.random.default_rng(100 * d + budget)
    for trial in range(3 if d < 10 else 1):
        e = rng.exponential(1.0, d // 2) * np.exp(rng.uniform(-4, 4, d // 2))
        g = allocation.greedy_bits(e, budget, d)
        opts, cost = _brute_force(e, budget)
        assert len(opts) == 1                  # distinct random energies: unique optimum
        assert tuple(g) == opts[0]
        assert allocation.allocation_cost(e, g, DIST) == pytest.approx(cost, rel=1e-15)


def test_ties_lower_index_and_optimal():
    e = np.array([1.0, 2.0, 2.0, 1.0])           # two tied pairs
    g = allocation.greedy_bits(e, 2, 8)
    opts, cost = _brute_force(e, 2)
    assert allocation.allocation_cost(e, g, DIST) == pytest.approx(cost, rel=1e-15)
    assert tuple(g) in opts
    # the odd bit of a tie goes to the lower index
    g1 = allocation.greedy_bits(np.array([1.0, 1.0]), 1, 4)   # 2 bits for 2 blocks of 2 dims
    assert g1.tolist() == [1, 1]
    g3 = allocation.greedy_bits(np.array([3.0, 3.0, 3.0]), 1, 6)
    assert g3.tolist() == [1, 1, 1]
    g5 = allocation.greedy_bits(np.array([5.0, 5.0]), 3, 4)    # 6 bits: 3 + 3
    assert g5.tolist() == [3, 3]


@pytest.mark.parametrize("budget", [1, 2, 3, 4, 5, 8])
def test_uniform_under_equal_energy(budget):
    g = allocation.greedy_bits(np.full(64, 0.37), budget, 128)
    assert g.tolist() == [budget] * 64


@pytest.mark.parametrize("budget", [2, 3])
def test_exact_budget_monotone_and_capped(budget):
    rng = np.random.default_rng(budget)
    for _ in range(20):
        e = np.exp(rng.uniform(-12, 6, 64))
        g = allocation.greedy_bits(e, budget, 128)
        assert 2 * int(g.sum()) == budget * 128
        assert g.max() <= 8 and g.min() >= 0
        order = np.argsort(-e)
        assert np.all(np.diff(g[order]) <= 0)        # E_i > E_j  =>  b_i >= b_j


def test_cap_binds():
    e = np.array([1e12] + [1e-12] * 7)
    g = allocation.greedy_bits(e, 4, 16)             # 64 bits -> 32 widths
    assert g[0] == 8 and int(g.sum()) == 32


def test_energy_definition_exact():
    rng = np.random.default_rng(5)
    k = (rng.standard_normal((37, 8)) * 3).astype(np.float16)
    e = allocation.block_energy(k, rope.HALF)
    for i in range(4):
        exact = sum(Fraction(float(x)) ** 2 for x in k[:, i]) + \
                sum(Fraction(float(x)) ** 2 for x in k[:, i + 4])
        assert e[i] == float(exact / 37)                 # correctly rounded mean


def test_groups_structure():
    bits = np.array([3, 0, 3, 1, 8, 1])
    gs = allocation.groups(bits, 12, rope.INTERLEAVED)
    assert [g.width for g in gs] == [1, 3, 8]
    assert gs[0].blocks == (3, 5) and gs[0].coords == (6, 7, 10, 11)
    assert gs[1].blocks == (0, 2) and gs[1].coords == (0, 1, 4, 5) and gs[1].m == 4
    gh = allocation.groups(bits, 12, rope.HALF)
    assert gh[1].coords == (0, 6, 2, 8)
    assert sum(g.m * g.width for g in gs) == 2 * int(bits.sum())
