"""gtq_block_energy_noalloc: the energy pass for callers that cannot allocate.

Some callers cannot call cudaMalloc when they need the energy pass (a CUDA
graph being captured, a server that reserved all device memory at start-up).
gtq_block_energy_noalloc runs the energy kernels with their scratch in a fixed
array inside the library.  These tests call it through the C ABI and check its
output against the energies of the allocating entry point (gtq_alloc_bits,
read back with gtq_get_energy) with the tolerance the other GPU tests use for
energies, on two calls in a row that share the fixed scratch.

This file runs last (pytest collects files alphabetically) and passes both on
its own in a fresh process and after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import decode_attention_13_b200 as gtq  # noqa: E402
from decode_attention_13_b200 import synth  # noqa: E402

pytestmark = pytest.mark.gpu

ENERGY_RTOL = 1e-12


def _energy_noalloc(cfg, k, T, stream=None):
    lib = gtq.binding.library()
    out = torch.full((cfg.batch, cfg.n_kv_heads, cfg.head_dim // 2), float("nan"),
                     dtype=torch.float64, device="cuda")
    st = (ctypes.c_int64 * 4)(*[int(v) for v in k.stride()])
    rc = lib.gtq_block_energy_noalloc(ctypes.byref(cfg), k.data_ptr(), int(T), st,
                                      out.data_ptr(),
                                      None if stream is None else stream.cuda_stream)
    return rc, out


def _energy_allocating(cfg, k, T):
    plan = gtq.gtq_alloc_bits(cfg, k, T)
    e = gtq.gtq_get_energy(plan)
    plan.free()
    return e


def _layer(seed, B, hkv, T, dtype):
    lay = synth.layer((seed,), B, hkv, 1, T, theta=1e4,
                      dtype=np.float16 if dtype == gtq.DTYPE_FP16 else np.float32)
    return torch.from_numpy(lay["k"]).cuda()


def test_two_calls_match_allocating_entry_point():
    cases = [(1, 2, 3000, gtq.DTYPE_FP16, 0), (2, 3, 1500, gtq.DTYPE_FP32, 1)]
    for B, hkv, T, dtype, pairing in cases:          # two calls in a row, shared scratch
        k = _layer(70 + T, B, hkv, T, dtype)
        cfg = gtq.make_config(B, hkv, hkv, 3, 3, T, in_dtype=dtype, rope_pairing=pairing)
        rc, e_static = _energy_noalloc(cfg, k, T)
        assert rc == gtq.GTQ_OK, gtq.strerror(rc)
        torch.cuda.synchronize()
        e_ref = _energy_allocating(cfg, k, T)
        got = e_static.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.allclose(got, e_ref, rtol=ENERGY_RTOL, atol=0)


def test_repeat_on_a_stream_gives_same_result():
    k = _layer(90, 1, 2, 2048, gtq.DTYPE_FP16)
    cfg = gtq.make_config(1, 2, 2, 3, 3, 2048)
    s = torch.cuda.Stream()
    rc1, e1 = _energy_noalloc(cfg, k, 2048, s)
    rc2, e2 = _energy_noalloc(cfg, k, 2048, s)
    s.synchronize()
    assert rc1 == rc2 == gtq.GTQ_OK
    assert torch.equal(e1, e2)


def test_rejects_sizes_beyond_the_fixed_scratch():
    # 64 heads x 65 chunks x 128 > 2^19 partial sums: rejected before any launch
    cfg = gtq.make_config(16, 4, 4, 3, 3, 66560)
    k = torch.zeros((1,), dtype=torch.float16, device="cuda")
    lib = gtq.binding.library()
    st = (ctypes.c_int64 * 4)(4 * 66560 * 128, 66560 * 128, 128, 1)
    out = torch.zeros((1,), dtype=torch.float64, device="cuda")
    rc = lib.gtq_block_energy_noalloc(ctypes.byref(cfg), k.data_ptr(), 66560, st,
                                      out.data_ptr(), None)
    assert rc == gtq.GTQ_ERR_UNSUPPORTED
    assert "fixed scratch" in lib.gtq_last_error().decode()
