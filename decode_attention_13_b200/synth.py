"""Seeded synthetic K/V/q inputs shaped like the models the Block-GTQ page measures.

This module only draws inputs; it holds none of Block-GTQ's arithmetic and is
shared by the tests, the benchmark and the smoke check.  The page evaluates
real models (Qwen2.5-3B-Instruct, Llama-3.1-8B-Instruct,
DeepSeek-R1-Distill-Qwen-7B; "RoPE-Aware Bit Allocation for KV-Cache
Quantization", Abstract) whose weights and prompts are not available, so keys
and queries are drawn with the RoPE-block structure those models show:

* per (layer, sequence, KV head): a decay rate a ~ U[1, 5] (or a fixed a) and
  two distinct outlier blocks drawn uniformly;
* pre-RoPE key block i ~ N(0, s_i^2 I_2) with s_i = exp(-a i / (d/2)), times 8
  on the two outlier blocks;
* each of the G query heads of that KV head: pre-RoPE block i ~ N(0, s_i^2 I_2)
  with the same s_i, drawn independently;
* values ~ N(0, 1);
* RoPE with w_i = theta^(-2i/d) at key positions 0..T-1 and query position T,
  in fp64, then a cast to the storage dtype (fp16, or fp32 for the small case).

``numpy`` draws (``head``) serve the CPU-sized cases; ``torch`` draws on a
device (``layer_torch``) follow the same recipe for the large workloads.  The
two paths use different random streams.
"""

from __future__ import annotations

import numpy as np

HALF = 0
INTERLEAVED = 1


def _pairs(d: int, pairing: int) -> np.ndarray:
    i = np.arange(d // 2)
    if pairing == HALF:
        return np.stack([i, i + d // 2], axis=1)
    return np.stack([2 * i, 2 * i + 1], axis=1)


def _apply_rope(x_blocks: np.ndarray, pos: np.ndarray, d: int, theta: float,
                pairing: int) -> np.ndarray:
    """x_blocks [n, d/2, 2] at positions pos [n] -> [n, d] (fp64)."""
    w = theta ** (-2.0 * np.arange(d // 2, dtype=np.float64) / d)
    ang = pos.astype(np.float64)[:, None] * w[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x_blocks[..., 0], x_blocks[..., 1]
    r0 = x0 * c - x1 * s
    r1 = x0 * s + x1 * c
    out = np.empty((x_blocks.shape[0], d))
    pr = _pairs(d, pairing)
    out[:, pr[:, 0]] = r0
    out[:, pr[:, 1]] = r1
    return out


def block_scales(d: int, a: float, outliers, outlier_scale: float = 8.0) -> np.ndarray:
    s = np.exp(-a * np.arange(d // 2) / (d // 2))
    s[list(outliers)] *= outlier_scale
    return s


def head(seed, T: int, d: int = 128, theta: float = 1e4, g_q: int = 1,
         decay: float | None = None, pairing: int = HALF, dtype=np.float16,
         outlier_scale: float = 8.0) -> dict:
    """One KV head: post-RoPE k [T, d], v [T, d], q [g_q, d] in ``dtype``.

    ``seed`` is an int or a tuple of ints (e.g. (config, layer, b, h)).
    Also returns the pre-RoPE k / q blocks (fp64) and the drawn parameters.
    """
    rng = np.random.default_rng(np.random.SeedSequence(seed))
    a = float(rng.uniform(1.0, 5.0)) if decay is None else float(decay)
    outl = rng.choice(d // 2, size=2, replace=False)
    s = block_scales(d, a, outl, outlier_scale)
    k_pre = rng.standard_normal((T, d // 2, 2)) * s[None, :, None]
    q_pre = rng.standard_normal((g_q, d // 2, 2)) * s[None, :, None]
    v = rng.standard_normal((T, d))
    k = _apply_rope(k_pre, np.arange(T), d, theta, pairing)
    q = _apply_rope(q_pre, np.full(g_q, T), d, theta, pairing)
    pr = _pairs(d, pairing)

    def flat(xb):
        out = np.empty((xb.shape[0], d))
        out[:, pr[:, 0]] = xb[..., 0]
        out[:, pr[:, 1]] = xb[..., 1]
        return out

    return {
        "k": k.astype(dtype), "v": v.astype(dtype), "q": q.astype(dtype),
        "k_pre": flat(k_pre), "q_pre": flat(q_pre), "a": a,
        "outliers": tuple(int(x) for x in outl), "theta": theta, "pairing": pairing,
    }


def layer(seed, B: int, h_kv: int, g_q: int, T: int, d: int = 128, theta: float = 1e4,
          decay: float | None = None, pairing: int = HALF, dtype=np.float16) -> dict:
    """A layer as numpy arrays: k, v [B, Hkv, T, d]; q [B, Hkv*g_q, d]."""
    seed = seed if isinstance(seed, tuple) else (seed,)
    k = np.empty((B, h_kv, T, d), dtype=dtype)
    v = np.empty((B, h_kv, T, d), dtype=dtype)
    q = np.empty((B, h_kv * g_q, d), dtype=dtype)
    for b in range(B):
        for h in range(h_kv):
            hd = head(seed + (b, h), T, d, theta, g_q, decay, pairing, dtype)
            k[b, h], v[b, h] = hd["k"], hd["v"]
            q[b, h * g_q:(h + 1) * g_q] = hd["q"]
    return {"k": k, "v": v, "q": q}


def layer_torch(seed, B: int, h_kv: int, g_q: int, T: int, d: int = 128,
                theta: float = 1e4, decay: float | None = None, pairing: int = HALF,
                dtype=None, device="cuda"):
    """Same recipe drawn with torch on ``device``: returns (k, v, q) tensors,
    k / v [B, Hkv, T, d] and q [B, Hkv*g_q, d] in ``dtype`` (default fp16)."""
    import torch

    dtype = torch.float16 if dtype is None else dtype
    seed = seed if isinstance(seed, tuple) else (seed,)
    ss = np.random.SeedSequence(seed)
    prm = np.random.default_rng(ss.spawn(1)[0])
    gen = torch.Generator(device=device)
    gen.manual_seed(int(ss.generate_state(1, dtype=np.uint64)[0] & 0x7FFFFFFFFFFFFFFF))
    k = torch.empty((B, h_kv, T, d), dtype=dtype, device=device)
    v = torch.empty((B, h_kv, T, d), dtype=dtype, device=device)
    q = torch.empty((B, h_kv * g_q, d), dtype=dtype, device=device)
    pr = _pairs(d, pairing)
    p0 = torch.as_tensor(pr[:, 0], device=device)
    p1 = torch.as_tensor(pr[:, 1], device=device)
    w = theta ** (-2.0 * torch.arange(d // 2, dtype=torch.float64, device=device) / d)
    pos_k = torch.arange(T, dtype=torch.float64, device=device)
    ang_k = pos_k[:, None] * w[None, :]
    ck, sk = torch.cos(ang_k), torch.sin(ang_k)
    ang_q = float(T) * w
    cq, sq = torch.cos(ang_q), torch.sin(ang_q)
    for b in range(B):
        for h in range(h_kv):
            a = float(prm.uniform(1.0, 5.0)) if decay is None else float(decay)
            outl = prm.choice(d // 2, size=2, replace=False)
            s = torch.as_tensor(block_scales(d, a, outl), device=device)
            kb = torch.randn((T, d // 2, 2), generator=gen, device=device,
                             dtype=torch.float64) * s[None, :, None]
            r0 = kb[..., 0] * ck - kb[..., 1] * sk
            r1 = kb[..., 0] * sk + kb[..., 1] * ck
            kk = torch.empty((T, d), dtype=torch.float64, device=device)
            kk[:, p0], kk[:, p1] = r0, r1
            k[b, h] = kk.to(dtype)
            v[b, h] = torch.randn((T, d), generator=gen, device=device,
                                  dtype=torch.float32).to(dtype)
            qb = torch.randn((g_q, d // 2, 2), generator=gen, device=device,
                             dtype=torch.float64) * s[None, :, None]
            q0 = qb[..., 0] * cq - qb[..., 1] * sq
            q1 = qb[..., 0] * sq + qb[..., 1] * cq
            qq = torch.empty((g_q, d), dtype=torch.float64, device=device)
            qq[:, p0], qq[:, p1] = q0, q1
            q[b, h * g_q:(h + 1) * g_q] = qq.to(dtype)
    return k, v, q


# Workloads (shapes of the page's models; the sizes the benchmark and tests use).
CONFIGS = {
    0: dict(name="single-head T=1024 fp32 K3V3", layers=1, B=1, h_q=1, h_kv=1, T=1024,
            theta=1e4, k_bits=3, v_bits=3, decay=3.0, dtype="fp32"),
    1: dict(name="Llama-3.1-8B-shaped layer 32q/8kv T=32768 K2V2", layers=1, B=1, h_q=32,
            h_kv=8, T=32768, theta=5e5, k_bits=2, v_bits=2, decay=None, dtype="fp16"),
    2: dict(name="Qwen2.5-3B-shaped 36 layers 16q/2kv T=131072 K3V3", layers=36, B=1,
            h_q=16, h_kv=2, T=131072, theta=1e6, k_bits=3, v_bits=3, decay=None,
            dtype="fp16"),
    3: dict(name="DeepSeek-R1-Distill-Qwen-7B-shaped 28 layers 28q/4kv B=16 T=16384 K3V2",
            layers=28, B=16, h_q=28, h_kv=4, T=16384, theta=1e4, k_bits=3, v_bits=2,
            decay=None, dtype="fp16"),
    4: dict(name="Qwen2.5-3B-shaped layer 16q/2kv T=524288 K3V3", layers=1, B=1, h_q=16,
            h_kv=2, T=524288, theta=1e6, k_bits=3, v_bits=3, decay=None, dtype="fp16"),
}
