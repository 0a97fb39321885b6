"""CPU checks of the test-side layout reader/writer: write -> read is the
identity on random codes, every bit of the code areas is used exactly once,
and the tile size matches the library's (via its host helper)."""
import numpy as np
import pytest

from tests import layout


@pytest.mark.parametrize("kb,vb,T", [(3, 3, 1), (3, 3, 130), (2, 2, 64), (3, 2, 100), (1, 8, 70), (8, 1, 65)])
def test_roundtrip(kb, vb, T):
    rng = np.random.default_rng(kb * 10 + vb + T)
    bits = np.zeros(64, np.int64)                      # random widths, exact budget
    while bits.sum() < kb * 64:
        i = rng.integers(0, 64)
        if bits[i] < 8:
            bits[i] += 1
    groups = layout.layout_groups(bits)
    keys = [(w, rng.integers(0, 2 ** w, (T, m)), rng.standard_normal(T).astype(np.float16))
            for (w, m) in groups]
    vc = rng.integers(0, 2 ** vb, (T, 128))
    vn = rng.standard_normal(T).astype(np.float16)
    n_tiles = (T + 63) // 64 + 1
    buf = layout.write_head(bits, keys, vc, vn, kb, vb, n_tiles)
    assert buf.size == n_tiles * layout.tile_bytes(kb, vb)
    k2, vc2, vn2 = layout.read_head(buf, bits, kb, vb, T)
    for (w, c, n16), (w2, c2, n2) in zip(keys, k2):
        assert w == w2 and np.array_equal(c, c2) and np.array_equal(n16, n2)
    assert np.array_equal(vc, vc2) and np.array_equal(vn, vn2)


def test_every_code_bit_used_once():
    bits = np.array([3] * 64)
    st = [s for (w, s0, jj, rr) in layout._key_maps(bits).values() for s in s0]
    spans = np.concatenate([np.arange(s, s + 3) for s in st])
    assert np.array_equal(np.sort(spans), np.arange(1024 * 3 * 8))
    s, jj, dd = layout._value_map(2)
    spans = np.concatenate([np.arange(x, x + 2) for x in s])
    assert np.array_equal(np.sort(spans), np.arange(1024 * 2 * 8))
    pairs = set(zip(jj.tolist(), dd.tolist()))
    assert len(pairs) == 64 * 128
