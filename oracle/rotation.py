"""Seeded orthogonal rotations R_m of TurboQuant-MSE (oracle, fp64).

TQ-MSE (the base quantizer of the allocator in "RoPE-Aware Bit Allocation for
KV-Cache Quantization", Abstract) rotates each normalised vector by a
fixed random orthogonal matrix so that every rotated coordinate is close to
N(0, 1/m), then codes sqrt(m) times each coordinate with the Lloyd-Max
quantizer of N(0, 1).

Construction read for this implementation (the page gives none):

* One matrix per size m (even, 2..128) for keys (tag 'K'), shared by every
  layer, head and sequence; one 128 x 128 matrix for values (tag 'V').
* Gaussian source: SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) used as a
  counter-based generator.  With gamma = 0x9E3779B97F4A7C15 and the published
  SplitMix64 output mix, the n-th 64-bit word of stream ``key`` is
  mix(key + (n + 1) * gamma  mod 2**64), key = seed ^ (tag << 48) ^ (m << 32).
* Entry (i, j) of the m x m Gaussian G (row-major n = i*m + j) takes words
  2n and 2n+1, forms u1 = ((w_{2n} >> 11) + 0.5) * 2**-53 in (0, 1) and
  u2 = (w_{2n+1} >> 11) * 2**-53, and is the Box-Muller cosine variate
  sqrt(-2 ln u1) * cos(2 pi u2).
* R_m = Q of the QR factorisation G = Q R, with the sign of each column of Q
  chosen so that diag(R) > 0 (the unique such factor).
"""

from __future__ import annotations

import functools

import numpy as np

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
_GAMMA = np.uint64(0x9E3779B97F4A7C15)
TAG_KEY = 0x4B    # 'K'
TAG_VALUE = 0x56  # 'V'


def splitmix64_words(key: int, count: int) -> np.ndarray:
    """Words 0..count-1 of the counter-based SplitMix64 stream ``key``."""
    with np.errstate(over="ignore"):
        n = np.arange(1, count + 1, dtype=np.uint64)
        z = np.uint64(key) + n * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def stream_key(seed: int, tag: int, m: int) -> int:
    return (int(seed) ^ (int(tag) << 48) ^ (int(m) << 32)) & 0xFFFFFFFFFFFFFFFF


def gaussian_matrix(m: int, tag: int, seed: int) -> np.ndarray:
    """The m x m standard-normal matrix G of stream (seed, tag, m)."""
    w = splitmix64_words(stream_key(seed, tag, m), 2 * m * m)
    u1 = ((w[0::2] >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53
    u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    two_pi = 2.0 * np.pi
    g = np.sqrt(-2.0 * np.log(u1)) * np.cos(two_pi * u2)
    return g.reshape(m, m)


@functools.lru_cache(maxsize=None)
def _rotation(m: int, tag: int, seed: int) -> np.ndarray:
    g = gaussian_matrix(m, tag, seed)
    q, r = np.linalg.qr(g)          # LAPACK Householder QR
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    q = q * s[None, :]              # columns scaled so that diag(R) > 0
    q.setflags(write=False)
    return q


def rotation(m: int, tag: int = TAG_KEY, seed: int = 0) -> np.ndarray:
    """R_m: the fixed seeded m x m orthogonal matrix (fp64, read-only)."""
    if m < 1:
        raise ValueError("m must be >= 1")
    return _rotation(int(m), int(tag), int(seed))


def key_rotation(m: int, seed: int = 0) -> np.ndarray:
    return rotation(m, TAG_KEY, seed)


def value_rotation(d: int = 128, seed: int = 0) -> np.ndarray:
    return rotation(d, TAG_VALUE, seed)
