"""Block-GTQ energy score, greedy bit allocation and block groups (oracle).

Per layer and KV head, Block-GTQ scores every RoPE block with an energy that
needs no labels, then hands out integer bit widths one at a time to the block
whose next bit gains the most ("RoPE-Aware Bit Allocation for KV-Cache
Quantization", Abstract).

Readings taken (the page prints no formula):

* Energy of block i over the T quantized post-RoPE keys of one (sequence,
  layer, KV head):  E_i = (1/T) sum_t (k_t[p0(i)]**2 + k_t[p1(i)]**2), in fp64.
  RoPE rotates each block, so E_i is the same before and after RoPE.
* Greedy: all b_i = 0; while sum_i 2 b_i < budget * d, give one bit to the
  block with the largest marginal gain E_i * (D(b_i) - D(b_i + 1)), where D is
  the Lloyd-Max distortion of N(0,1); ties go to the lower index (first
  strictly greater gain in ascending i); blocks at max_bits (8) are not
  eligible.  The loop ends with sum_i 2 b_i = budget * d exactly.
* Groups: the blocks of equal nonzero width w form one group, members in
  ascending block order; its coordinates are listed block by block, p0 then
  p1, so the group has m = 2 * (number of blocks) coordinates.  Width-0 blocks
  store nothing and contribute 0 to the logit.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from . import lloyd_max, rope

MAX_BITS = 8


def block_energy(k: np.ndarray, pairing: int = rope.HALF) -> np.ndarray:
    """E_i for one head: k is [T, d] (post-RoPE, any float dtype).

    Each square of an fp16/fp32 input is exact in fp64; the sum over tokens is
    the correctly rounded fp64 sum (math.fsum), divided by T in fp64.
    """
    k = np.asarray(k)
    T, d = k.shape
    bd = rope.block_dims(d, pairing)
    kk = k.astype(np.float64)
    e = np.empty(d // 2)
    for i in range(d // 2):
        sq = np.concatenate([kk[:, bd[i, 0]] ** 2, kk[:, bd[i, 1]] ** 2])
        e[i] = math.fsum(sq.tolist()) / T
    return e


def greedy_bits(energy: np.ndarray, budget_bits: int, d: int | None = None,
                max_bits: int = MAX_BITS, dist: np.ndarray | None = None) -> np.ndarray:
    """Integer width b_i of every block by greedy marginal gain (fp64)."""
    energy = np.asarray(energy, dtype=np.float64)
    n = energy.shape[0]
    if d is None:
        d = 2 * n
    if dist is None:
        dist = lloyd_max.distortion_table(max_bits)
    target = budget_bits * d
    b = [0] * n
    total = 0
    while total < target:
        best, best_gain = -1, 0.0
        for i in range(n):
            if b[i] >= max_bits:
                continue
            gain = float(energy[i]) * (float(dist[b[i]]) - float(dist[b[i] + 1]))
            if best < 0 or gain > best_gain:
                best, best_gain = i, gain
        if best < 0:
            raise ValueError("budget exceeds max_bits on every block")
        b[best] += 1
        total += 2
    return np.array(b, dtype=np.int64)


def allocation_cost(energy: np.ndarray, bits: np.ndarray, dist: np.ndarray) -> float:
    """sum_i E_i D(b_i): the distortion the greedy allocation minimises."""
    return float(sum(float(e) * float(dist[int(b)]) for e, b in zip(energy, bits)))


@dataclass(frozen=True)
class Group:
    width: int
    blocks: tuple      # ascending block indices
    coords: tuple      # head dims, block by block, p0 then p1

    @property
    def m(self) -> int:
        return len(self.coords)


def groups(bits: np.ndarray, d: int, pairing: int = rope.HALF) -> list:
    """Groups of equal nonzero width, in ascending width order.

    (The order of groups is a listing convention only; no quantity depends on it.)
    """
    bd = rope.block_dims(d, pairing)
    out = []
    for w in sorted(set(int(x) for x in bits if int(x) > 0)):
        blocks = tuple(int(i) for i in range(len(bits)) if int(bits[i]) == w)
        coords = tuple(int(c) for i in blocks for c in bd[i])
        out.append(Group(width=w, blocks=blocks, coords=coords))
    return out
