"""Pins for the RoPE facts: the post-RoPE logit equals the sum of its per-block
terms and depends on positions only through T - t; RoPE keeps block energy."""
import numpy as np
import pytest

from decode_attention_13_b200 import synth
from oracle import allocation, rope


@pytest.mark.parametrize("pairing", [rope.HALF, rope.INTERLEAVED])
def test_logit_is_sum_of_block_terms(pairing):
    hd = synth.head((7,), T=64, d=128, theta=1e4, g_q=1, pairing=pairing, dtype=np.float64)
    T = 64
    for t in (0, 5, 63):
        full = float(hd["q"][0] @ hd["k"][t])
        terms = rope.per_block_logits(hd["q_pre"][0], hd["k_pre"][t], T, t, 1e4, pairing)
        assert terms.shape == (64,)
        assert full == pytest.approx(float(np.sum(terms)), abs=1e-10)


def test_block_terms_depend_on_offset_only():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    a = rope.per_block_logits(q, k, T=100, t=37, theta=500.0)
    b = rope.per_block_logits(q, k, T=1100, t=1037, theta=500.0)
    assert np.allclose(a, b, atol=1e-9)
    c = rope.per_block_logits(q, k, T=100, t=38, theta=500.0)
    assert not np.allclose(a, c, atol=1e-6)


@pytest.mark.parametrize("pairing", [rope.HALF, rope.INTERLEAVED])
def test_energy_invariant_under_rope(pairing):
    hd = synth.head((3,), T=256, d=128, theta=1e6, pairing=pairing, dtype=np.float64)
    e_post = allocation.block_energy(hd["k"], pairing)
    e_pre = allocation.block_energy(hd["k_pre"], pairing)
    assert np.allclose(e_post, e_pre, rtol=1e-12, atol=0)


def test_block_dims():
    assert rope.block_dims(8, rope.HALF).tolist() == [[0, 4], [1, 5], [2, 6], [3, 7]]
    assert rope.block_dims(8, rope.INTERLEAVED).tolist() == [[0, 1], [2, 3], [4, 5], [6, 7]]
