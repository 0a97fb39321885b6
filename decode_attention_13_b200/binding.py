"""ctypes binding of libgtq (the C ABI in include/gtq.h).

Argument marshalling only: every step of the hot path runs in the CUDA library
(``libgtq.so``, built in-tree by ``decode_attention_13_b200.build``).  There is
no Python or CPU fallback: importing this package raises if the library is
missing, and every wrapper raises ``GtqError`` on a nonzero return code.

The functions mirror the C ABI in ``include/gtq.h``:

    plan = gtq_alloc_bits(cfg, k, T, stream=None)          # energy + greedy
    gtq_quantize_pack(plan, k, v, t0, n, packed, stream=None)
    gtq_decode_attn(plan, packed, T, q, out, stream=None)
    gtq_free(plan)

Tensor arguments may be torch tensors (CUDA memory; their data pointer and
strides are passed through) or raw integer device pointers.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgtq.so")

GTQ_OK = 0
GTQ_T0_TAIL = -1  # gtq_quantize_pack_ex: write the last n tokens of every sequence
GTQ_ERR_INVALID = -1
GTQ_ERR_UNSUPPORTED = -2
GTQ_ERR_CUDA = -3
GTQ_ERR_OOM = -4
GTQ_ERR_TIMEOUT = -5
GTQ_ERR_OVERFLOW = -6
GTQ_ERR_STATE = -7
PAIRING_HALF = 0
PAIRING_INTERLEAVED = 1
DTYPE_FP16 = 0
DTYPE_FP32 = 1
TILE_TOKENS = 64
TAG_KEY = 0x4B
TAG_VALUE = 0x56

ABI_FUNCTIONS = (
    "gtq_alloc_bits", "gtq_alloc_bits_from_energy", "gtq_quantize_pack", "gtq_decode_attn",
    "gtq_free", "gtq_packed_bytes", "gtq_get_bits", "gtq_get_energy", "gtq_status",
    "gtq_strerror", "gtq_last_error", "gtq_lloyd_max", "gtq_rotation", "gtq_layout_tile_bytes",
    "gtq_block_energy_noalloc", "gtq_plan_device_bytes", "gtq_raise_status",
    "gtq_alloc_bits_ex", "gtq_quantize_pack_ex", "gtq_decode_attn_ex", "gtq_decode_attn_full",
)


class GtqError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = ""
        if code in (GTQ_ERR_CUDA, GTQ_ERR_OOM):
            detail = " [%s]" % _lib.gtq_last_error().decode()
        super().__init__("%s failed: %s (%d)%s" % (where, strerror(code), code, detail))


class gtq_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("k_bits", ctypes.c_int32), ("v_bits", ctypes.c_int32),
        ("max_bits", ctypes.c_int32), ("rope_pairing", ctypes.c_int32),
        ("in_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("seed", ctypes.c_uint64), ("t_capacity", ctypes.c_int64),
    ]


class gtq_seq_layout(ctypes.Structure):
    _fields_ = [
        ("seq_lens_dev", ctypes.c_void_p), ("block_table_dev", ctypes.c_void_p),
        ("max_blocks", ctypes.c_int64),
    ]


def seq_layout(seq_lens=None, block_table=None):
    """A gtq_seq_layout from device int32 tensors: lengths [batch] and a block
    table [batch][max_blocks] (either may be None).  Keep the tensors alive
    while the calls that use the layout run."""
    lay = gtq_seq_layout(None, None, 0)
    if seq_lens is not None:
        lay.seq_lens_dev = _ptr(seq_lens)
    if block_table is not None:
        lay.block_table_dev = _ptr(block_table)
        lay.max_blocks = int(block_table.shape[1])
    return lay


class gtq_fp16_kv(ctypes.Structure):
    _fields_ = [
        ("v_dev", ctypes.c_void_p), ("v_strides", ctypes.c_int64 * 4),
        ("recent_k_dev", ctypes.c_void_p), ("recent_v_dev", ctypes.c_void_p),
        ("recent_strides", ctypes.c_int64 * 4), ("recent_lens_dev", ctypes.c_void_p),
        ("recent_len", ctypes.c_int64),
    ]


def fp16_kv(v=None, recent_k=None, recent_v=None, recent_lens=None, recent_len=None):
    """A gtq_fp16_kv from device fp16 tensors: values [batch, kv_heads, tokens, 128]
    of a K-only plan, and a window of recent keys / values [batch, kv_heads, rows,
    128] (same strides for both) with optional int32 lengths [batch].  Keep the
    tensors alive while the calls that use it run."""
    kv = gtq_fp16_kv()
    if v is not None:
        kv.v_dev = _ptr(v)
        kv.v_strides = (ctypes.c_int64 * 4)(*[int(s) for s in v.stride()])
    if recent_k is not None:
        if tuple(recent_k.stride()) != tuple(recent_v.stride()):
            raise ValueError("recent keys and values must share strides")
        kv.recent_k_dev = _ptr(recent_k)
        kv.recent_v_dev = _ptr(recent_v)
        kv.recent_strides = (ctypes.c_int64 * 4)(*[int(s) for s in recent_k.stride()])
        kv.recent_len = int(recent_k.shape[2]) if recent_len is None else int(recent_len)
    if recent_lens is not None:
        kv.recent_lens_dev = _ptr(recent_lens)
    return kv


def make_config(batch, n_q_heads, n_kv_heads, k_bits, v_bits, t_capacity, head_dim=128,
                max_bits=8, rope_pairing=PAIRING_HALF, in_dtype=DTYPE_FP16, seed=0) -> gtq_config:
    return gtq_config(batch, n_q_heads, n_kv_heads, head_dim, k_bits, v_bits, max_bits,
                      rope_pairing, in_dtype, 0, seed, t_capacity)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libgtq.so not built (run `python -m decode_attention_13_b200.build`); "
                          "there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    I64x4 = ctypes.POINTER(ctypes.c_int64)
    sig = {
        "gtq_alloc_bits": (I32, [ctypes.POINTER(gtq_config), P, I64, I64x4, P, ctypes.POINTER(P)]),
        "gtq_alloc_bits_from_energy": (I32, [ctypes.POINTER(gtq_config), ctypes.POINTER(ctypes.c_double), ctypes.POINTER(P)]),
        "gtq_quantize_pack": (I32, [P, P, P, I64x4, I64, I64, P, SZ, P]),
        "gtq_decode_attn": (I32, [P, P, I64, P, I32, P, P]),
        "gtq_free": (I32, [P]),
        "gtq_packed_bytes": (SZ, [P]),
        "gtq_get_bits": (I32, [P, ctypes.POINTER(ctypes.c_uint8), P]),
        "gtq_get_energy": (I32, [P, ctypes.POINTER(ctypes.c_double), P]),
        "gtq_status": (I32, [P]),
        "gtq_strerror": (ctypes.c_char_p, [I32]),
        "gtq_last_error": (ctypes.c_char_p, []),
        "gtq_lloyd_max": (I32, [I32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
        "gtq_rotation": (I32, [ctypes.c_uint64, I32, I32, ctypes.POINTER(ctypes.c_double)]),
        "gtq_layout_tile_bytes": (SZ, [I32, I32]),
        "gtq_block_energy_noalloc": (I32, [ctypes.POINTER(gtq_config), P, I64, I64x4, P, P]),
        "gtq_plan_device_bytes": (SZ, [P]),
        "gtq_raise_status": (I32, [P, I32]),
        "gtq_alloc_bits_ex": (I32, [ctypes.POINTER(gtq_config), P, I64, I64x4,
                                    ctypes.POINTER(gtq_seq_layout), P, ctypes.POINTER(P)]),
        "gtq_quantize_pack_ex": (I32, [P, P, P, I64x4, I64, I64, P, SZ,
                                       ctypes.POINTER(gtq_seq_layout), P]),
        "gtq_decode_attn_ex": (I32, [P, P, I64, ctypes.POINTER(gtq_seq_layout), P, I32, P, P]),
        "gtq_decode_attn_full": (I32, [P, P, I64, ctypes.POINTER(gtq_seq_layout),
                                       ctypes.POINTER(gtq_fp16_kv), P, I32, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


_lib = _load()


def library():
    """The loaded ctypes library (for ABI checks)."""
    return _lib


def strerror(code: int) -> str:
    return _lib.gtq_strerror(int(code)).decode()


def _check(rc: int, where: str) -> None:
    if rc != GTQ_OK:
        raise GtqError(rc, where)


def _ptr(x) -> int:
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(s) -> int:
    if s is None:
        return 0
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def _strides4(x, strides):
    if strides is not None:
        return (ctypes.c_int64 * 4)(*[int(v) for v in strides])
    st = tuple(int(v) for v in x.stride())
    if len(st) != 4:
        raise ValueError("K/V must be 4-D [batch, kv_heads, tokens, head_dim]")
    return (ctypes.c_int64 * 4)(*st)


class Plan:
    """Owning handle of a gtq_plan (freed by gtq_free or on garbage collection)."""

    def __init__(self, handle: int, cfg: gtq_config):
        self.handle = handle
        self.cfg = cfg

    @property
    def packed_bytes(self) -> int:
        return int(_lib.gtq_packed_bytes(self.handle))

    def free(self) -> None:
        if self.handle:
            h, self.handle = self.handle, None
            _check(_lib.gtq_free(h), "gtq_free")

    def __del__(self):
        try:
            if self.handle:
                _lib.gtq_free(self.handle)
        except Exception:
            pass


def gtq_alloc_bits(cfg: gtq_config, k, T: int, stream=None, strides=None) -> Plan:
    out = ctypes.c_void_p()
    rc = _lib.gtq_alloc_bits(ctypes.byref(cfg), _ptr(k), int(T), _strides4(k, strides),
                             _stream(stream), ctypes.byref(out))
    _check(rc, "gtq_alloc_bits")
    return Plan(out.value, cfg)


def gtq_alloc_bits_from_energy(cfg: gtq_config, energy) -> Plan:
    import numpy as np

    e = np.ascontiguousarray(energy, dtype=np.float64)
    out = ctypes.c_void_p()
    rc = _lib.gtq_alloc_bits_from_energy(ctypes.byref(cfg),
                                         e.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                         ctypes.byref(out))
    _check(rc, "gtq_alloc_bits_from_energy")
    return Plan(out.value, cfg)


def gtq_quantize_pack(plan: Plan, k, v, t0: int, n_tokens: int, packed, stream=None,
                      strides=None, packed_bytes=None) -> None:
    nbytes = packed_bytes if packed_bytes is not None else (
        packed.numel() * packed.element_size())
    rc = _lib.gtq_quantize_pack(plan.handle, _ptr(k), _ptr(v), _strides4(k, strides), int(t0),
                                int(n_tokens), _ptr(packed), int(nbytes), _stream(stream))
    _check(rc, "gtq_quantize_pack")


def gtq_decode_attn(plan: Plan, packed, T: int, q, out, stream=None, q_dtype=None) -> None:
    if q_dtype is None:
        import torch

        q_dtype = DTYPE_FP32 if q.dtype == torch.float32 else DTYPE_FP16
    rc = _lib.gtq_decode_attn(plan.handle, _ptr(packed), int(T), _ptr(q), int(q_dtype),
                              _ptr(out), _stream(stream))
    _check(rc, "gtq_decode_attn")


def _lay(layout):
    return None if layout is None else ctypes.byref(layout)


def gtq_alloc_bits_ex(cfg: gtq_config, k, T: int, layout=None, stream=None,
                      strides=None) -> Plan:
    out = ctypes.c_void_p()
    rc = _lib.gtq_alloc_bits_ex(ctypes.byref(cfg), _ptr(k), int(T), _strides4(k, strides),
                                _lay(layout), _stream(stream), ctypes.byref(out))
    _check(rc, "gtq_alloc_bits_ex")
    return Plan(out.value, cfg)


def gtq_quantize_pack_ex(plan: Plan, k, v, t0: int, n_tokens: int, packed, layout=None,
                         stream=None, strides=None, packed_bytes=None) -> None:
    nbytes = packed_bytes if packed_bytes is not None else (
        packed.numel() * packed.element_size())
    rc = _lib.gtq_quantize_pack_ex(plan.handle, _ptr(k), _ptr(v), _strides4(k, strides),
                                   int(t0), int(n_tokens), _ptr(packed), int(nbytes),
                                   _lay(layout), _stream(stream))
    _check(rc, "gtq_quantize_pack_ex")


def gtq_decode_attn_ex(plan: Plan, packed, T: int, q, out, layout=None, stream=None,
                       q_dtype=None) -> None:
    if q_dtype is None:
        import torch

        q_dtype = DTYPE_FP32 if q.dtype == torch.float32 else DTYPE_FP16
    rc = _lib.gtq_decode_attn_ex(plan.handle, _ptr(packed), int(T), _lay(layout), _ptr(q),
                                 int(q_dtype), _ptr(out), _stream(stream))
    _check(rc, "gtq_decode_attn_ex")


def gtq_decode_attn_full(plan: Plan, packed, T: int, q, out, layout=None, kv=None, stream=None,
                         q_dtype=None) -> None:
    if q_dtype is None:
        import torch

        q_dtype = DTYPE_FP32 if q.dtype == torch.float32 else DTYPE_FP16
    rc = _lib.gtq_decode_attn_full(plan.handle, _ptr(packed), int(T), _lay(layout),
                                   None if kv is None else ctypes.byref(kv), _ptr(q),
                                   int(q_dtype), _ptr(out), _stream(stream))
    _check(rc, "gtq_decode_attn_full")


def gtq_free(plan: Plan) -> None:
    plan.free()


def gtq_packed_bytes(plan: Plan) -> int:
    return plan.packed_bytes


def gtq_get_bits(plan: Plan, stream=None):
    import numpy as np

    c = plan.cfg
    out = np.zeros((c.batch, c.n_kv_heads, c.head_dim // 2), dtype=np.uint8)
    _check(_lib.gtq_get_bits(plan.handle, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                             _stream(stream)), "gtq_get_bits")
    return out


def gtq_get_energy(plan: Plan, stream=None):
    import numpy as np

    c = plan.cfg
    out = np.zeros((c.batch, c.n_kv_heads, c.head_dim // 2), dtype=np.float64)
    _check(_lib.gtq_get_energy(plan.handle, out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                               _stream(stream)), "gtq_get_energy")
    return out


def gtq_status(plan: Plan) -> int:
    return int(_lib.gtq_status(plan.handle))


def gtq_plan_device_bytes(plan: Plan) -> int:
    return int(_lib.gtq_plan_device_bytes(plan.handle))


def gtq_raise_status(plan: Plan, code: int) -> None:
    _check(_lib.gtq_raise_status(plan.handle, int(code)), "gtq_raise_status")


def gtq_lloyd_max(bits: int):
    import numpy as np

    c = np.zeros(1 << bits)
    t = np.zeros(max(1, (1 << bits) - 1))
    d = ctypes.c_double()
    _check(_lib.gtq_lloyd_max(int(bits), c.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                              t.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), ctypes.byref(d)),
           "gtq_lloyd_max")
    return c, t[: (1 << bits) - 1], d.value


def gtq_rotation(m: int, tag: int = TAG_KEY, seed: int = 0):
    import numpy as np

    out = np.zeros((m, m))
    _check(_lib.gtq_rotation(int(seed), int(tag), int(m),
                             out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))), "gtq_rotation")
    return out


def gtq_layout_tile_bytes(k_bits: int, v_bits: int) -> int:
    return int(_lib.gtq_layout_tile_bytes(int(k_bits), int(v_bits)))
