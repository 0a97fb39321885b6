"""CPU checks of the C ABI (no GPU calls): the library loads, exports every
function include/gtq.h declares, its host tables match the oracle, and
argument validation rejects bad calls before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import decode_attention_13_b200 as gtq
from oracle import lloyd_max, rotation

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "gtq.h")).read()
    return set(re.findall(r"GTQ_API\s+[\w\s\*]+?\b(gtq_\w+)\s*\(", text))


def test_header_and_binding_agree():
    assert _declared() == set(gtq.binding.ABI_FUNCTIONS)


def test_every_declared_symbol_exported():
    lib = ctypes.CDLL(gtq.binding.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_library_lloyd_max_matches_oracle():
    for b in range(0, 9):
        c, t, d = gtq.gtq_lloyd_max(b)
        assert np.max(np.abs(c - lloyd_max.centroids(b))) < 1e-12
        if b:
            assert np.max(np.abs(t - lloyd_max.thresholds(b))) < 1e-12
            assert np.array_equal(t.astype(np.float32), lloyd_max.thresholds(b).astype(np.float32))
        assert abs(d - lloyd_max.distortion(b)) < 1e-15


def test_library_rotations_match_oracle():
    for seed in (0, 7):
        for m in (2, 4, 18, 64, 128):
            assert np.max(np.abs(gtq.gtq_rotation(m, gtq.TAG_KEY, seed) - rotation.key_rotation(m, seed))) < 1e-12
        assert np.max(np.abs(gtq.gtq_rotation(128, gtq.TAG_VALUE, seed) - rotation.value_rotation(128, seed))) < 1e-12


def test_tile_bytes():
    assert gtq.gtq_layout_tile_bytes(3, 3) == 1024 * 6 + 128 + 1024
    assert gtq.gtq_layout_tile_bytes(0, 3) == 0


def _cfg(**kw):
    base = dict(batch=1, n_q_heads=8, n_kv_heads=2, k_bits=3, v_bits=3, t_capacity=1024)
    base.update(kw)
    return gtq.make_config(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), gtq.GTQ_ERR_INVALID),
    (dict(n_q_heads=7), gtq.GTQ_ERR_INVALID),
    (dict(n_q_heads=258), gtq.GTQ_ERR_UNSUPPORTED),     # GQA group of 129
    (dict(batch=32768, n_q_heads=4), gtq.GTQ_ERR_UNSUPPORTED),  # 65536 KV heads
    (dict(batch=1 << 30, n_q_heads=4), gtq.GTQ_ERR_UNSUPPORTED),  # int overflow of B * Hkv
    (dict(head_dim=130), gtq.GTQ_ERR_UNSUPPORTED),
    (dict(head_dim=12), gtq.GTQ_ERR_UNSUPPORTED),       # alloc from K needs a multiple of 8
    (dict(k_bits=0), gtq.GTQ_ERR_INVALID),
    (dict(k_bits=9), gtq.GTQ_ERR_INVALID),
    (dict(v_bits=9), gtq.GTQ_ERR_INVALID),
    (dict(rope_pairing=2), gtq.GTQ_ERR_INVALID),
    (dict(in_dtype=3), gtq.GTQ_ERR_INVALID),
    (dict(t_capacity=0), gtq.GTQ_ERR_INVALID),
])
def test_alloc_rejects_bad_config(kw, code):
    cfg = _cfg(**kw)
    st = (ctypes.c_int64 * 4)(2 * 1024 * 128, 1024 * 128, 128, 1)
    out = ctypes.c_void_p()
    rc = gtq.binding._lib.gtq_alloc_bits(ctypes.byref(cfg), 0x1000, 16, st, None, ctypes.byref(out))
    assert rc == code and out.value is None


def test_alloc_rejects_bad_pointers_and_sizes():
    lib = gtq.binding._lib
    cfg = _cfg()
    st = (ctypes.c_int64 * 4)(2 * 1024 * 128, 1024 * 128, 128, 1)
    out = ctypes.c_void_p()
    assert lib.gtq_alloc_bits(None, 0x1000, 16, st, None, ctypes.byref(out)) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_alloc_bits(ctypes.byref(cfg), None, 16, st, None, ctypes.byref(out)) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_alloc_bits(ctypes.byref(cfg), 0x1002, 16, st, None, ctypes.byref(out)) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_alloc_bits(ctypes.byref(cfg), 0x1000, 0, st, None, ctypes.byref(out)) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_alloc_bits(ctypes.byref(cfg), 0x1000, 2048, st, None, ctypes.byref(out)) == gtq.GTQ_ERR_INVALID
    bad = (ctypes.c_int64 * 4)(2 * 1024 * 128, 1024 * 128, 128, 2)
    assert lib.gtq_alloc_bits(ctypes.byref(cfg), 0x1000, 16, bad, None, ctypes.byref(out)) == gtq.GTQ_ERR_INVALID
    odd = (ctypes.c_int64 * 4)(2 * 1024 * 128, 1024 * 128, 129, 1)
    assert lib.gtq_alloc_bits(ctypes.byref(cfg), 0x1000, 16, odd, None, ctypes.byref(out)) == gtq.GTQ_ERR_INVALID
    assert out.value is None


def test_null_plan_calls():
    lib = gtq.binding._lib
    st = (ctypes.c_int64 * 4)(0, 0, 128, 1)
    assert lib.gtq_quantize_pack(None, 0x1000, 0x1000, st, 0, 1, 0x1000, 1 << 20, None) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_decode_attn(None, 0x1000, 1, 0x1000, 0, 0x1000, None) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_free(None) == gtq.GTQ_OK
    assert lib.gtq_packed_bytes(None) == 0
    assert lib.gtq_status(None) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_get_bits(None, None, None) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_lloyd_max(9, None, None, None) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_rotation(0, 0x4B, 3, None) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_rotation(0, 0x41, 4, (ctypes.c_double * 16)()) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_rotation(0, 0x56, 64, (ctypes.c_double * 4096)()) == gtq.GTQ_ERR_INVALID


def test_strerror_names():
    for code in range(-7, 1):
        assert gtq.strerror(code) and gtq.strerror(code) != "unknown error"
    assert gtq.strerror(-99) == "unknown error"


def test_noalloc_energy_rejects_head_count_overflow():
    # batch * n_kv_heads is formed in 64 bits and bounded by the grid limit
    # (65535) before any device call, so this runs without a GPU
    lib = gtq.binding._lib
    st = (ctypes.c_int64 * 4)(0, 0, 128, 1)
    for batch, hkv in ((65536, 1), (1 << 20, 1 << 12), (2 ** 31 - 1, 2 ** 31 - 1)):
        cfg = gtq.make_config(batch, hkv, hkv, 3, 3, 64)
        rc = lib.gtq_block_energy_noalloc(ctypes.byref(cfg), 0x1000, 64, st, 0x1000, None)
        assert rc == gtq.GTQ_ERR_INVALID
        assert "65535" in lib.gtq_last_error().decode()


def test_status_helpers_reject_null_plan():
    lib = gtq.binding._lib
    assert lib.gtq_raise_status(None, gtq.GTQ_ERR_TIMEOUT) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_plan_device_bytes(None) == 0


def test_key_only_tile_bytes_and_reader_agree():
    from tests import layout

    for kb in range(1, 9):
        assert gtq.gtq_layout_tile_bytes(kb, 0) == 1024 * kb + 1024 == layout.tile_bytes(kb, 0)
        for vb in range(1, 9):
            assert gtq.gtq_layout_tile_bytes(kb, vb) == layout.tile_bytes(kb, vb)
    assert gtq.gtq_layout_tile_bytes(3, 9) == 0 and gtq.gtq_layout_tile_bytes(3, -1) == 0


def test_null_plan_calls_of_the_layout_entry_points():
    lib = gtq.binding._lib
    st = (ctypes.c_int64 * 4)(0, 0, 128, 1)
    lay = gtq.binding.gtq_seq_layout(None, None, 0)
    kv = gtq.binding.gtq_fp16_kv()
    out = ctypes.c_void_p()
    assert lib.gtq_alloc_bits_ex(None, 0x1000, 1, st, ctypes.byref(lay), None,
                                 ctypes.byref(out)) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_quantize_pack_ex(None, 0x1000, 0x1000, st, 0, 1, 0x1000, 1 << 20,
                                    ctypes.byref(lay), None) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_decode_attn_ex(None, 0x1000, 1, ctypes.byref(lay), 0x1000, 0, 0x1000,
                                  None) == gtq.GTQ_ERR_INVALID
    assert lib.gtq_decode_attn_full(None, 0x1000, 1, None, ctypes.byref(kv), 0x1000, 0, 0x1000,
                                    None) == gtq.GTQ_ERR_INVALID


def test_struct_layouts_match_the_header():
    # the binding's ctypes structs against the C compiler's view of include/gtq.h
    import shutil
    import subprocess
    import tempfile

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = {
        "gtq_config": [f for f, _ in gtq.binding.gtq_config._fields_],
        "gtq_seq_layout": [f for f, _ in gtq.binding.gtq_seq_layout._fields_],
        "gtq_fp16_kv": [f for f, _ in gtq.binding.gtq_fp16_kv._fields_],
    }
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "gtq.h"', 'int main(void) {']
    for st, fs in fields.items():
        lines.append('printf("%s %%zu\\n", sizeof(%s));' % (st, st))
        for f in fs:
            lines.append('printf("%s.%s %%zu\\n", offsetof(%s, %s));' % (st, f, st, f))
    lines += ['return 0;', '}']
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "t.c"), os.path.join(d, "t")
        open(src, "w").write("\n".join(lines))
        subprocess.run([cc, "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True)
        got = dict(l.split() for l in subprocess.run([exe], capture_output=True, text=True,
                                                    check=True).stdout.split("\n") if l)
    for st, fs in fields.items():
        cls = getattr(gtq.binding, st)
        assert int(got[st]) == ctypes.sizeof(cls), st
        for f in fs:
            assert int(got["%s.%s" % (st, f)]) == getattr(cls, f).offset, (st, f)
