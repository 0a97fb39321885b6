"""TurboQuant-MSE group coding of keys and values (oracle, fp64).

Block-GTQ codes keys with TurboQuant-MSE (TQ-MSE) as the base quantizer and is
compared against TQ-MSE with one width for every block, at the same K/V bit
budgets ("RoPE-Aware Bit Allocation for KV-Cache Quantization", Abstract).

Construction read for this implementation:

* Keys, per token and per group g (width w, m coords, rotation R_m):
  n = ||k_g|| in fp64; if n = 0 the norm is 0 and every code is 0; otherwise
  y = sqrt(m) * R_m k_g / n and code_j = number of w-bit Lloyd-Max thresholds
  below y_j.  The stored norm is fp16(n), round-to-nearest-even, clamped to
  65504 (norms above that are flagged).  The exact fp64 n scales y; the fp16
  norm is only stored and used at decode.
* Values: uniform TQ-MSE over the whole head, i.e. one group of all d coords
  in natural order, width b_V, rotation R_V (tag 'V').
* Uniform TQ-MSE keys (the comparison arm): one group of all d coords, listed
  block by block (p0 then p1), width b_K, rotation R_d (tag 'K').
* Dequantised vector of a group: k_hat_g = R_m^T (fp16(n) / sqrt(m)) cb_w[code].
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import allocation, lloyd_max, rotation

FP16_MAX = 65504.0


@dataclass
class CodedGroup:
    width: int
    coords: tuple          # head dims of the group, in coding order
    codes: np.ndarray      # [T, m] int64, logical row order of R_m
    norm16: np.ndarray     # [T] float16 stored norm
    norm64: np.ndarray     # [T] float64 exact norm
    overflow: bool         # some norm exceeded the fp16 range

    @property
    def m(self) -> int:
        return len(self.coords)


def code_group(x: np.ndarray, width: int, rot: np.ndarray,
               decision_dtype=np.float32) -> tuple:
    """Code rows of x [T, m] with one rotation; returns (codes, norm16, norm64, overflow)."""
    x = np.asarray(x, dtype=np.float64)
    T, m = x.shape
    n = np.sqrt(np.sum(x * x, axis=1))
    codes = np.zeros((T, m), dtype=np.int64)
    nz = n > 0
    if np.any(nz):
        y = np.sqrt(m) * (x[nz] @ rot.T) / n[nz][:, None]
        codes[nz] = lloyd_max.encode(y, width, decision_dtype)
    overflow = bool(np.any(n > FP16_MAX))
    norm16 = np.minimum(n, FP16_MAX).astype(np.float16)
    return codes, norm16, n, overflow


def quantize_keys(k: np.ndarray, bits: np.ndarray, pairing: int, seed: int = 0,
                  decision_dtype=np.float32) -> list:
    """Block-GTQ key codes of one head: k [T, d] post-RoPE, bits [d/2]."""
    k = np.asarray(k)
    d = k.shape[1]
    out = []
    for g in allocation.groups(bits, d, pairing):
        rot = rotation.key_rotation(g.m, seed)
        codes, n16, n64, ovf = code_group(k[:, list(g.coords)], g.width, rot, decision_dtype)
        out.append(CodedGroup(g.width, g.coords, codes, n16, n64, ovf))
    return out


def quantize_keys_uniform(k: np.ndarray, k_bits: int, pairing: int, seed: int = 0,
                          decision_dtype=np.float32) -> list:
    """Uniform TQ-MSE key codes: one group of all d coords at k_bits each."""
    d = np.asarray(k).shape[1]
    bits = np.full(d // 2, k_bits, dtype=np.int64)
    return quantize_keys(k, bits, pairing, seed, decision_dtype)


def quantize_values(v: np.ndarray, v_bits: int, seed: int = 0,
                    decision_dtype=np.float32) -> CodedGroup:
    """Uniform TQ-MSE value codes of one head: v [T, d]."""
    v = np.asarray(v)
    d = v.shape[1]
    rot = rotation.value_rotation(d, seed)
    codes, n16, n64, ovf = code_group(v, v_bits, rot, decision_dtype)
    return CodedGroup(v_bits, tuple(range(d)), codes, n16, n64, ovf)


def dequantize_group(g: CodedGroup, rot: np.ndarray) -> np.ndarray:
    """[T, m] reconstruction of the group's coordinates in the original basis."""
    cb = lloyd_max.decode(g.codes, g.width)                       # [T, m]
    scaled = cb * (g.norm16.astype(np.float64) / np.sqrt(g.m))[:, None]
    return scaled @ rot                                           # R^T applied per row


def dequantize_keys(groups_: list, d: int, T: int, seed: int = 0) -> np.ndarray:
    """k_hat [T, d]; dims of width-0 blocks are 0."""
    out = np.zeros((T, d))
    for g in groups_:
        out[:, list(g.coords)] = dequantize_group(g, rotation.key_rotation(g.m, seed))
    return out


def dequantize_values(g: CodedGroup, seed: int = 0) -> np.ndarray:
    return dequantize_group(g, rotation.value_rotation(g.m, seed))
