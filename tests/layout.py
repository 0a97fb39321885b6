"""Independent numpy reader / writer of libgtq's packed-cache layout (version 1).

Written from the layout description in include/gtq.h only (it shares no code
with the CUDA library).  The tests use it to
  * read the library's packed cache back into logical codes and norms, and
  * write the oracle's codes into the layout, so that the GPU decode and the
    oracle decode run on identical packed inputs.

Logical form of one head (as in oracle.quantize): for every nonzero-width group
(width w, m rows of R_m) a codes array [T, m] in row order and an fp16 norm
array [T]; values: codes [T, 128] (rows of R_V) and fp16 norms [T].
Layout groups are listed in DESCENDING width.
"""

from __future__ import annotations

import numpy as np

TILE = 64


def tile_bytes(kb: int, vb: int) -> int:
    """vb = 0: keys only (no value codes and no value norms)."""
    return 1024 * (kb + vb) + (128 if vb else 0) + 128 * 8


def _knorm(kb: int, vb: int) -> int:
    return 1024 * (kb + vb) + (128 if vb else 0)


def layout_groups(bits) -> list:
    """(width, m) of every nonzero-width group, descending width."""
    out = []
    for w in range(8, 0, -1):
        cnt = int(np.sum(np.asarray(bits) == w))
        if cnt:
            out.append((w, 2 * cnt))
    return out


def _key_maps(bits):
    """Per width: (bit start in the tile's key area, token j, group, row) of every code."""
    maps = {}
    off = 0
    for gi, (w, m) in enumerate(layout_groups(bits)):
        st, jj, gg, rr = [], [], [], []
        for rp in range(m // 2):
            for g in range(8):
                for u in range(8):
                    for e in range(2):
                        st.append(off * 8 + g * 16 * w + (2 * u + e) * w)
                        jj.append(g + 8 * u)
                        gg.append(gi)
                        rr.append(2 * rp + e)
            off += 16 * w
        maps[gi] = (w, np.array(st), np.array(jj), np.array(rr))
    return maps


def _value_map(vb):
    st, jj, dd = [], [], []
    for p in range(256):
        i, g, c4 = p >> 5, (p >> 2) & 7, p & 3
        for x in range(32):
            dd.append(16 * i + g + 8 * ((x >> 1) & 1))
            jj.append(16 * (x >> 3) + 2 * c4 + (x & 1) + 8 * ((x >> 2) & 1))
            st.append(p * 32 * vb + x * vb)
    return np.array(st), np.array(jj), np.array(dd)


def _norm_map():
    g, u = np.meshgrid(np.arange(8), np.arange(8), indexing="ij")
    return (g + 8 * u).ravel()          # token of entry [g][u], row-major


def _gather(bitmat, starts, w):
    v = np.zeros((bitmat.shape[0], len(starts)), np.int64)
    for k in range(w):
        v |= bitmat[:, starts + k].astype(np.int64) << k
    return v


def _scatter(bitmat, starts, vals, w):
    for k in range(w):
        bitmat[:, starts + k] = (vals >> k) & 1


def read_head(buf: np.ndarray, bits, kb: int, vb: int, T: int):
    """buf: uint8 bytes of one head (>= ceil(T/64) tiles).  Returns
    (keys: list of (width, codes [T, m], norm16 [T]) descending width,
     vcodes [T, 128], vnorm16 [T])."""
    tb = tile_bytes(kb, vb)
    n = (T + TILE - 1) // TILE
    tiles = np.asarray(buf[:n * tb], np.uint8).reshape(n, tb)
    groups = layout_groups(bits)
    kbits = np.unpackbits(tiles[:, :1024 * kb], axis=1, bitorder="little")
    vbits = np.unpackbits(tiles[:, 1024 * kb:1024 * (kb + vb)], axis=1, bitorder="little")
    tok = (np.arange(n) * TILE)[:, None]
    keys = []
    for gi, (w, st, jj, rr) in _key_maps(bits).items():
        codes = np.zeros((n * TILE, groups[gi][1]), np.int64)
        codes[(tok + jj[None, :]).ravel(), np.tile(rr, n)] = _gather(kbits, st, w).ravel()
        nm = tiles[:, _knorm(kb, vb) + gi * 128:][:, :128].copy().view(np.float16)
        n16 = np.zeros(n * TILE, np.float16)
        n16[(tok + _norm_map()[None, :]).ravel()] = nm.ravel()
        keys.append((w, codes[:T], n16[:T]))
    if vb == 0:
        return keys, None, None
    st, jj, dd = _value_map(vb)
    vcodes = np.zeros((n * TILE, 128), np.int64)
    vcodes[(tok + jj[None, :]).ravel(), np.tile(dd, n)] = _gather(vbits, st, vb).ravel()
    vn = tiles[:, 1024 * (kb + vb):1024 * (kb + vb) + 128].copy().view(np.float16)
    vnorm = np.zeros(n * TILE, np.float16)
    vnorm[(tok + _norm_map()[None, :]).ravel()] = vn.ravel()
    return keys, vcodes[:T], vnorm[:T]


def write_head(bits, key_groups: list, vcodes: np.ndarray, vnorm16: np.ndarray, kb: int, vb: int,
               n_tiles: int) -> np.ndarray:
    """Inverse of read_head (tokens >= T of the last tile are zero).
    key_groups: list of (width, codes [T, m], norm16 [T]) in descending width."""
    tb = tile_bytes(kb, vb)
    T = (vcodes.shape[0] if vcodes is not None else np.asarray(key_groups[0][1]).shape[0])
    n = (T + TILE - 1) // TILE
    assert [w for (w, _) in layout_groups(bits)] == [g[0] for g in key_groups]
    pad = n * TILE - T

    def padrows(a):
        return np.concatenate([a, np.zeros((pad,) + a.shape[1:], a.dtype)]) if pad else a

    tok = (np.arange(n) * TILE)[:, None]
    kbits = np.zeros((n, 1024 * kb * 8), np.uint8)
    for gi, (w, st, jj, rr) in _key_maps(bits).items():
        codes = padrows(np.asarray(key_groups[gi][1], np.int64))
        vals = codes[(tok + jj[None, :]), rr[None, :]]
        _scatter(kbits, st, vals, w)
    out = np.zeros((n_tiles, tb), np.uint8)
    out[:n, :1024 * kb] = np.packbits(kbits, axis=1, bitorder="little")
    nmap = _norm_map()
    if vb:
        st, jj, dd = _value_map(vb)
        vbits = np.zeros((n, 1024 * vb * 8), np.uint8)
        vc = padrows(np.asarray(vcodes, np.int64))
        _scatter(vbits, st, vc[(tok + jj[None, :]), dd[None, :]], vb)
        out[:n, 1024 * kb:1024 * (kb + vb)] = np.packbits(vbits, axis=1, bitorder="little")
        vn = padrows(np.asarray(vnorm16, np.float16))[(tok + nmap[None, :])]
        o = 1024 * (kb + vb)
        out[:n, o:o + 128] = vn.view(np.uint8).reshape(n, 128)
    o = _knorm(kb, vb)
    for gi, (w, codes, n16) in enumerate(key_groups):
        kn = padrows(np.asarray(n16, np.float16))[(tok + nmap[None, :])]
        out[:n, o + gi * 128:o + 128 + gi * 128] = kn.view(np.uint8).reshape(n, 128)
    return out.ravel()


def gather_paged_head(pool: np.ndarray, table_row, hkv: int, h: int, n_tiles: int,
                      tb: int) -> np.ndarray:
    """The n_tiles tiles of KV head h of one sequence, read from a paged pool
    (page p holds one tile of every KV head: head h at (p * hkv + h) tiles),
    concatenated in token order as a contiguous head buffer."""
    out = np.empty(n_tiles * tb, np.uint8)
    for n in range(n_tiles):
        off = (int(table_row[n]) * hkv + h) * tb
        out[n * tb:(n + 1) * tb] = pool[off:off + tb]
    return out
