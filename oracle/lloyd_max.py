"""Lloyd-Max scalar quantizer of a standard normal variable (oracle, fp64).

Block-GTQ takes TurboQuant-MSE (TQ-MSE) as its base quantizer ("RoPE-Aware
Bit Allocation for KV-Cache Quantization", Abstract).  TQ-MSE codes each rotated, normalised
coordinate with the MSE-optimal (Lloyd-Max) scalar quantizer of N(0, 1), and
Block-GTQ's marginal gain of one more bit on a block is measured with that
quantizer's distortion D(b).

A b-bit Lloyd-Max quantizer has N = 2**b reconstruction levels (centroids)
c_0 < ... < c_{N-1} and N-1 decision thresholds t_1 < ... < t_{N-1}; it is the
fixed point of the two optimality conditions

    t_k = (c_{k-1} + c_k) / 2                                  (nearest level)
    c_k = E[X | t_k < X < t_{k+1}]
        = (phi(t_k) - phi(t_{k+1})) / (Phi(t_{k+1}) - Phi(t_k)) (centroid)

with t_0 = -inf, t_N = +inf, phi / Phi the N(0,1) density / distribution.  At
the fixed point the mean squared error is D(b) = 1 - sum_k P_k c_k**2 with
P_k = Phi(t_{k+1}) - Phi(t_k).  D(0) = 1 (a single level at 0).

Reading taken: codes are numbered in increasing centroid order, and a value
lying exactly on a threshold takes the lower code (code = number of thresholds
strictly below the value).
"""

from __future__ import annotations

import functools
import warnings

import numpy as np
from scipy.optimize import fsolve
from scipy.special import ndtr, ndtri

_SQRT_2PI = np.sqrt(2.0 * np.pi)


def _phi(x: np.ndarray) -> np.ndarray:
    """N(0,1) density, 0 at +-inf."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    fin = np.isfinite(x)
    out[fin] = np.exp(-0.5 * x[fin] * x[fin]) / _SQRT_2PI
    return out


def cell_probability(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """P(a < X < b) for X ~ N(0,1), evaluated on the side of 0 that has no
    cancellation (upper-tail difference when a >= 0)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.where(a >= 0, ndtr(-a) - ndtr(-b), ndtr(b) - ndtr(a))


def centroids_for_thresholds(t: np.ndarray) -> np.ndarray:
    """Centroid condition: conditional mean of N(0,1) in every cell."""
    a = np.concatenate([[-np.inf], t])
    b = np.concatenate([t, [np.inf]])
    return (_phi(a) - _phi(b)) / cell_probability(a, b)


def thresholds_for_centroids(c: np.ndarray) -> np.ndarray:
    """Nearest-level condition: midpoints of adjacent centroids."""
    return 0.5 * (c[1:] + c[:-1])


@functools.lru_cache(maxsize=None)
def _solve(b: int):
    if b == 0:
        return np.zeros(1), np.zeros(0), 1.0
    n = 2 ** b
    # start: the companding (high-resolution) placement sqrt(3)*Phi^-1((k+1/2)/N)
    c = np.sqrt(3.0) * ndtri((np.arange(n) + 0.5) / n)
    # Lloyd's alternation of the two conditions ...
    for _ in range(200):
        c = centroids_for_thresholds(thresholds_for_centroids(c))
    # ... finished by a root solve of c = centroid(midpoints(c)) (MINPACK hybrd),
    # which reaches the fixed point that plain alternation approaches slowly.
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        c = fsolve(lambda x: x - centroids_for_thresholds(thresholds_for_centroids(x)),
                   c, xtol=1e-15)
    for _ in range(20):
        c = centroids_for_thresholds(thresholds_for_centroids(c))
    # N(0,1) is symmetric, so the optimal quantizer is: c_k = -c_{N-1-k}
    # (makes the middle threshold exactly 0 instead of a rounding residue)
    c = 0.5 * (c - c[::-1])
    t = thresholds_for_centroids(c)
    p = cell_probability(np.concatenate([[-np.inf], t]), np.concatenate([t, [np.inf]]))
    d = 1.0 - float(np.sum(p * c * c))
    return c, t, d


def centroids(b: int) -> np.ndarray:
    """The 2**b reconstruction levels, ascending (code k -> centroids(b)[k])."""
    return _solve(int(b))[0].copy()


def thresholds(b: int) -> np.ndarray:
    """The 2**b - 1 decision thresholds, ascending."""
    return _solve(int(b))[1].copy()


def distortion(b: int) -> float:
    """D(b): MSE of the b-bit Lloyd-Max quantizer on N(0,1); D(0) = 1."""
    return _solve(int(b))[2]


def distortion_table(max_bits: int) -> np.ndarray:
    """[D(0), D(1), ..., D(max_bits)]."""
    return np.array([distortion(b) for b in range(max_bits + 1)], dtype=np.float64)


def optimality_residual(b: int) -> float:
    """max |c - centroid(midpoints(c))| at the solution (0 at the exact fixed point)."""
    c = centroids(b)
    return float(np.max(np.abs(c - centroids_for_thresholds(thresholds_for_centroids(c)))))


def encode(y: np.ndarray, b: int, decision_dtype=np.float32) -> np.ndarray:
    """Code of each value: number of thresholds strictly below it.

    The comparison is taken in ``decision_dtype`` (both the value and the
    threshold rounded to it).  float32 is the precision the GPU quantizer decides
    in; pass np.float64 for the exact-arithmetic decision.
    """
    if b == 0:
        return np.zeros(np.shape(y), dtype=np.int64)
    t = thresholds(b).astype(decision_dtype)
    yy = np.asarray(y).astype(decision_dtype)
    return np.searchsorted(t, yy, side="left").astype(np.int64)


def decode(codes: np.ndarray, b: int) -> np.ndarray:
    """Reconstruction level of each code (fp64)."""
    return centroids(b)[np.asarray(codes, dtype=np.int64)]
