"""CPU fp64 oracle for Block-GTQ (test infrastructure, not the product).

This package is the plain, slow, obviously-correct statement of what the
Block-GTQ hot path computes.  It exists to check the CUDA library: only the
test-suite, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg
and its ``--impl reference`` arm) may import it.  It shares no code, tables or
constants with ``decode_attention_13_b200`` (the CUDA library and its binding),
and the library never imports it.

Source: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (Liang, Zhang,
Jia; arXiv 2606.24033), Abstract.  The abstract names the pieces -- the RoPE
2-D block decomposition of a key's logit contribution, a label-free energy per
RoPE block, greedy integer bit allocation by marginal gain per layer and KV
head, TurboQuant-MSE (TQ-MSE) as the base quantizer, and a packed-cache decode
path -- but prints no formula.  Every construction detail is stated where it is
used, with the reading taken where the page is silent.

Modules
-------
lloyd_max   b-bit Lloyd-Max scalar quantizer of N(0,1): centroids, thresholds, D(b)
rotation    seeded m x m orthogonal matrices (QR of a counter-based Gaussian)
rope        RoPE 2-D block pairing and the per-block logit decomposition
allocation  per-block energy, greedy marginal-gain bit allocation, block groups
quantize    TurboQuant-MSE group coding of keys and values (and the uniform arm)
attention   GQA decode attention on the codes, by two independent routes

Every function is pinned by a ``-m "not gpu"`` test against facts that do not
come from this package (closed forms, brute force, invariants, printed values).
"""

from . import lloyd_max, rotation, rope, allocation, quantize, attention  # noqa: F401
