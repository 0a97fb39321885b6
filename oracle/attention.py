"""GQA decode attention over Block-GTQ codes (oracle, fp64).

The page reports decoding straight from the packed K/V cache at serving time
("RoPE-Aware Bit Allocation for KV-Cache Quantization", Abstract).
The construction read for it: the logit uses the dequantised keys, and since
every group's rotation is orthogonal it can be taken in the rotated basis,

    s_t = (1/sqrt(d)) * sum_g (fp16(n_tg) / sqrt(m_g)) * (R_g q_g) . cb_wg[c_tg]

then p = softmax over the T cached tokens t = 0..T-1 (the query at position T
attends to the cached keys only: no mask, no self key), and

    o = R_V^T  sum_t p_t (fp16(n_Vt) / sqrt(d)) cb_bV[c_Vt]

i.e. P.V accumulated in V's rotated basis with R_V^T applied once.  The scale
1/sqrt(d) is standard attention's (reading: the construction leaves it implicit).

Two independent routes are provided; they must agree to rounding:
``decode_rotated`` (the formulas above) and ``decode_dequantised`` (rebuild
k_hat, v_hat in the original basis, then textbook softmax(q.k_hat/sqrt(d)).V_hat).
"""

from __future__ import annotations

import numpy as np

from . import lloyd_max, quantize, rotation


def _softmax(s: np.ndarray) -> np.ndarray:
    s = s - np.max(s, axis=-1, keepdims=True)
    e = np.exp(s)
    return e / np.sum(e, axis=-1, keepdims=True)


def decode_rotated(q: np.ndarray, key_groups: list, values: quantize.CodedGroup,
                   seed: int = 0) -> np.ndarray:
    """q [G, d] (the G query heads of one KV head) -> out [G, d] fp64."""
    q = np.asarray(q, dtype=np.float64)
    G, d = q.shape
    T = values.codes.shape[0]
    s = np.zeros((G, T))
    for g in key_groups:
        r = rotation.key_rotation(g.m, seed)
        qg = q[:, list(g.coords)] @ r.T                       # [G, m] = R_g q_g
        cb = lloyd_max.decode(g.codes, g.width)               # [T, m]
        s += (qg @ cb.T) * (g.norm16.astype(np.float64) / np.sqrt(g.m))[None, :]
    s /= np.sqrt(d)
    p = _softmax(s)                                           # [G, T]
    cbv = lloyd_max.decode(values.codes, values.width)        # [T, d]
    o_rot = p @ (cbv * (values.norm16.astype(np.float64) / np.sqrt(d))[:, None])
    return o_rot @ rotation.value_rotation(d, seed)          # rows: (R_V^T o_rot)^T


def decode_dequantised(q: np.ndarray, key_groups: list, values: quantize.CodedGroup,
                       seed: int = 0) -> np.ndarray:
    """Same result via explicit k_hat, v_hat in the original basis."""
    q = np.asarray(q, dtype=np.float64)
    G, d = q.shape
    T = values.codes.shape[0]
    k_hat = quantize.dequantize_keys(key_groups, d, T, seed)
    v_hat = quantize.dequantize_values(values, seed)
    p = _softmax(q @ k_hat.T / np.sqrt(d))
    return p @ v_hat


def attention_exact(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Unquantised softmax(q.k/sqrt(d)).v in fp64 (for context and tests)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    return _softmax(q @ k.T / np.sqrt(q.shape[1])) @ v


def logit_mae(q: np.ndarray, k: np.ndarray, k_hat: np.ndarray) -> float:
    """Mean |q.k_hat - q.k| over queries and tokens (unscaled RoPE logits)."""
    q = np.asarray(q, dtype=np.float64)
    return float(np.mean(np.abs(q @ np.asarray(k_hat, np.float64).T
                                - q @ np.asarray(k, np.float64).T)))


def decode_general(q: np.ndarray, key_groups: list, values=None, v_fp16=None,
                   k_recent=None, v_recent=None, seed: int = 0) -> np.ndarray:
    """Decode over coded keys with either coded values or fp16 values (the
    page's K-only quantization, Abstract), plus an optional window of recent
    tokens kept in fp16 (the fp16 recent-key buffer the page's method does
    without, Abstract).

    Reading taken: the query attends to the T coded tokens and then to the W
    window tokens in one softmax; window logits are q . k / sqrt(d) with the
    exact fp16 keys, window values are the exact fp16 values.  With K-only
    values, P.V uses the T exact fp16 value rows (no rotation).  Returns [G, d].
    """
    q = np.asarray(q, dtype=np.float64)
    G, d = q.shape
    T = (values.codes.shape[0] if values is not None else np.asarray(v_fp16).shape[0])
    s = np.zeros((G, T))
    for g in key_groups:
        r = rotation.key_rotation(g.m, seed)
        qg = q[:, list(g.coords)] @ r.T
        cb = lloyd_max.decode(g.codes, g.width)
        s += (qg @ cb.T) * (g.norm16.astype(np.float64) / np.sqrt(g.m))[None, :]
    s /= np.sqrt(d)
    if values is not None:
        cbv = lloyd_max.decode(values.codes, values.width)
        v_rows = (cbv * (values.norm16.astype(np.float64) / np.sqrt(d))[:, None]) \
            @ rotation.value_rotation(d, seed)                      # R_V^T per row
    else:
        v_rows = np.asarray(v_fp16, dtype=np.float64)
    if k_recent is not None and len(k_recent):
        kr = np.asarray(k_recent, dtype=np.float64)
        s = np.concatenate([s, q @ kr.T / np.sqrt(d)], axis=1)
        v_rows = np.concatenate([v_rows, np.asarray(v_recent, dtype=np.float64)], axis=0)
    return _softmax(s) @ v_rows
