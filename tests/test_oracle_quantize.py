"""Pins for oracle.quantize: fp16 norm rounding, zero vectors, distortion of the
TQ-MSE coder against D(b), and code range."""
import numpy as np
import pytest

from decode_attention_13_b200 import synth
from oracle import allocation, lloyd_max, quantize, rotation, rope


def test_norm_fp16_round_to_nearest_even_from_fp64():
    # 1 + 2^-11 + 2^-40 lies just above the midpoint between fp16 1.0 and
    # 1 + 2^-10: correct rounding goes up; rounding through fp32 first would
    # land exactly on the midpoint and go to even (down).
    x = 1 + 2.0 ** -11 + 2.0 ** -40
    codes, n16, n64, ovf = quantize.code_group(np.array([[x, 0.0]]), 2, rotation.key_rotation(2))
    assert float(n16[0]) == 1 + 2.0 ** -10
    assert not ovf


def test_zero_vector_codes_zero():
    codes, n16, n64, ovf = quantize.code_group(np.zeros((3, 4)), 3, rotation.key_rotation(4))
    assert np.all(codes == 0) and np.all(n16 == 0)


def test_overflow_clamped_and_flagged():
    codes, n16, n64, ovf = quantize.code_group(np.array([[7e4, 0.0]]), 1, rotation.key_rotation(2))
    assert ovf and float(n16[0]) == 65504.0


@pytest.mark.parametrize("w", [1, 2, 3, 4])
def test_group_distortion_matches_lloyd_max(w):
    # For random directions, sqrt(m) R x/|x| has coordinates close to N(0,1):
    # the relative squared error of the reconstruction is close to D(w).
    rng = np.random.default_rng(w)
    m = 128
    x = rng.standard_normal((4000, m))
    rot = rotation.key_rotation(m, 0)
    codes, n16, n64, _ = quantize.code_group(x, w, rot, np.float64)
    g = quantize.CodedGroup(w, tuple(range(m)), codes, n16, n64, False)
    xh = quantize.dequantize_group(g, rot)
    rel = np.sum((x - xh) ** 2) / np.sum(x ** 2)
    assert rel == pytest.approx(lloyd_max.distortion(w), rel=0.03)


def test_key_groups_cover_budget_and_code_range():
    hd = synth.head((11,), T=300, d=128, theta=1e4, dtype=np.float16)
    e = allocation.block_energy(hd["k"], rope.HALF)
    bits = allocation.greedy_bits(e, 3, 128)
    gs = quantize.quantize_keys(hd["k"], bits, rope.HALF)
    assert sum(g.m * g.width for g in gs) == 3 * 128
    for g in gs:
        assert g.codes.min() >= 0 and g.codes.max() < 2 ** g.width
        assert g.codes.shape == (300, g.m)
    v = quantize.quantize_values(hd["v"], 3)
    assert v.codes.shape == (300, 128) and v.codes.max() < 8


def test_fp32_decision_close_to_fp64():
    hd = synth.head((12,), T=500, d=128, theta=1e4, dtype=np.float16)
    bits = allocation.greedy_bits(allocation.block_energy(hd["k"]), 3, 128)
    a = quantize.quantize_keys(hd["k"], bits, rope.HALF, decision_dtype=np.float32)
    b = quantize.quantize_keys(hd["k"], bits, rope.HALF, decision_dtype=np.float64)
    diff = sum(int(np.sum(x.codes != y.codes)) for x, y in zip(a, b))
    tot = sum(x.codes.size for x in a)
    assert diff / tot < 1e-4
    for x, y in zip(a, b):
        assert np.all(np.abs(x.codes - y.codes) <= 1)
