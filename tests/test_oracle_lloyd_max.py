"""Pins for oracle.lloyd_max: closed forms, a printed table, optimality,
symmetry, the high-resolution limit and Monte Carlo distortion."""
import json
import math
import os

import numpy as np
import pytest

from oracle import lloyd_max

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_one_bit_closed_form():
    # 1-bit optimum for N(0,1): levels +-E|X| = +-sqrt(2/pi), threshold 0,
    # D = 1 - 2/pi (textbook closed form)
    c = lloyd_max.centroids(1)
    assert np.allclose(c, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-15)
    assert lloyd_max.thresholds(1)[0] == pytest.approx(0.0, abs=1e-15)
    assert lloyd_max.distortion(1) == pytest.approx(1 - 2 / math.pi, abs=1e-15)


def test_zero_bit():
    assert lloyd_max.distortion(0) == 1.0
    assert list(lloyd_max.centroids(0)) == [0.0]


def test_max_1960_table():
    g = json.load(open(os.path.join(GOLDEN, "lloyd_max_max1960.json")))
    for e in g["entries"]:
        b = e["bits"]
        c = lloyd_max.centroids(b)
        pos = c[2 ** (b - 1):]
        assert np.allclose(pos, e["positive_levels"], atol=e["level_tol"]), (b, pos)
        assert abs(lloyd_max.distortion(b) - e["distortion"]) <= e["distortion_tol"], b


@pytest.mark.parametrize("b", range(1, 9))
def test_optimality_and_symmetry(b):
    c = lloyd_max.centroids(b)
    t = lloyd_max.thresholds(b)
    assert len(c) == 2 ** b and len(t) == 2 ** b - 1
    assert np.all(np.diff(c) > 0)
    assert lloyd_max.optimality_residual(b) < 1e-13
    assert np.allclose(t, 0.5 * (c[1:] + c[:-1]), atol=0, rtol=0)
    assert np.allclose(c, -c[::-1], atol=1e-13)


def test_distortion_via_quadrature():
    # D(b) = sum_k int_{cell k} (x - c_k)^2 phi(x) dx, evaluated by adaptive
    # quadrature independently of the closed-form D = 1 - sum P_k c_k^2.
    from scipy.integrate import quad
    for b in (2, 3, 5):
        c = lloyd_max.centroids(b)
        edges = np.concatenate([[-np.inf], lloyd_max.thresholds(b), [np.inf]])
        pdf = lambda x: math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
        tot = 0.0
        for k in range(len(c)):
            tot += quad(lambda x: (x - c[k]) ** 2 * pdf(x), edges[k], edges[k + 1],
                        epsabs=1e-14, epsrel=1e-12)[0]
        assert tot == pytest.approx(lloyd_max.distortion(b), abs=1e-11)


def test_high_resolution_limit():
    # Panter-Dite: D(b) * 4^b -> pi*sqrt(3)/2 for a Gaussian, from below
    lim = math.pi * math.sqrt(3) / 2
    r = [lloyd_max.distortion(b) * 4 ** b for b in range(1, 9)]
    assert all(x < y for x, y in zip(r, r[1:]))
    assert r[-1] < lim and lim - r[-1] < 0.03


def test_distortion_convex():
    # marginal gains D(b) - D(b+1) strictly decrease: greedy allocation is optimal
    d = lloyd_max.distortion_table(8)
    gains = d[:-1] - d[1:]
    assert np.all(np.diff(gains) < 0)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_monte_carlo_mse(b):
    rng = np.random.default_rng(b)
    x = rng.standard_normal(2_000_000)
    xh = lloyd_max.decode(lloyd_max.encode(x, b, np.float64), b)
    mse = float(np.mean((x - xh) ** 2))
    assert mse == pytest.approx(lloyd_max.distortion(b), rel=0.01)


@pytest.mark.parametrize("b", [1, 2, 3, 5, 8])
def test_threshold_count_is_nearest_level(b):
    rng = np.random.default_rng(10 + b)
    y = rng.standard_normal(20000) * 1.5
    c = lloyd_max.centroids(b)
    nearest = np.argmin(np.abs(y[:, None] - c[None, :]), axis=1)
    assert np.array_equal(lloyd_max.encode(y, b, np.float64), nearest)


def test_encode_tie_goes_low():
    t = lloyd_max.thresholds(2)
    assert lloyd_max.encode(np.array([t[1]]), 2, np.float64)[0] == 1
    assert lloyd_max.encode(np.array([np.nextafter(t[1], 10)]), 2, np.float64)[0] == 2
