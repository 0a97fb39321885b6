"""RoPE 2-D frequency blocks and the block decomposition of a logit (oracle).

With RoPE, the part of a future attention logit that a key contributes splits
into a sum of terms, one per two-dimensional frequency block, each depending on
the relative position ("RoPE-Aware Bit Allocation for KV-Cache Quantization",
Abstract).

With frequencies w_i = theta**(-2 i / d), i = 0..d/2-1, RoPE rotates the 2-D
block i of a vector at position p by the angle p * w_i.  For a query at
position T and a key at position t, the logit is

    q_T . k_t = sum_i  q_i^T  Rot((t - T) w_i)  k_i                (*)

where q_i, k_i are the pre-RoPE blocks: every term depends on the positions
only through t - T.

Reading taken for the block pairing (the page says only "two-dimensional
frequency blocks"): HALF pairs dims (i, i + d/2) -- the rotate-half convention
of the Llama / Qwen models the page evaluates -- and is the default;
INTERLEAVED pairs dims (2i, 2i + 1).  Plain RoPE, no frequency scaling.
"""

from __future__ import annotations

import numpy as np

HALF = 0
INTERLEAVED = 1


def block_dims(d: int, pairing: int = HALF) -> np.ndarray:
    """[d/2, 2] array: the two dims (p0, p1) of every RoPE block."""
    if d % 2:
        raise ValueError("head_dim must be even")
    i = np.arange(d // 2)
    if pairing == HALF:
        return np.stack([i, i + d // 2], axis=1)
    if pairing == INTERLEAVED:
        return np.stack([2 * i, 2 * i + 1], axis=1)
    raise ValueError("unknown pairing")


def frequencies(d: int, theta: float) -> np.ndarray:
    return theta ** (-2.0 * np.arange(d // 2, dtype=np.float64) / d)


def rot2(angle: float) -> np.ndarray:
    c, s = np.cos(angle), np.sin(angle)
    return np.array([[c, -s], [s, c]])


def per_block_logits(q_pre: np.ndarray, k_pre: np.ndarray, T: int, t: int,
                     theta: float, pairing: int = HALF) -> np.ndarray:
    """The d/2 terms q_i^T Rot((t - T) w_i) k_i of (*) from pre-RoPE vectors."""
    d = q_pre.shape[-1]
    bd = block_dims(d, pairing)
    w = frequencies(d, theta)
    out = np.empty(d // 2)
    for i in range(d // 2):
        qi = q_pre[bd[i]].astype(np.float64)
        ki = k_pre[bd[i]].astype(np.float64)
        out[i] = qi @ rot2((t - T) * w[i]) @ ki
    return out
