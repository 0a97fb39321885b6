"""Block-GTQ packed KV cache for NVIDIA B200 (sm_100a).

The hot path lives in the CUDA library ``libgtq.so`` (C ABI: ``include/gtq.h``).
Its Python binding is ``decode_attention_13_b200.binding``; the ABI functions
(``gtq_alloc_bits``, ``gtq_quantize_pack``, ``gtq_decode_attn``, ``gtq_free``
and helpers) are re-exported here on first access, which loads the library
and raises ImportError if it has not been built -- there is no fallback.

``decode_attention_13_b200.synth`` (seeded synthetic inputs) does not load the
library.
"""

__all__ = ["binding", "synth", "build"]


def __getattr__(name):
    import importlib

    if name in ("synth", "build", "binding"):
        return importlib.import_module("." + name, __name__)
    binding = importlib.import_module(".binding", __name__)
    try:
        return getattr(binding, name)
    except AttributeError:
        raise AttributeError("module %r has no attribute %r" % (__name__, name)) from None
