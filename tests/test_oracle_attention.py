"""Pins for oracle.attention: two independent routes agree, degenerate cases
reduce to closed forms, high-rate codes approach exact attention, and Block-GTQ
keeps logits closer than uniform TQ-MSE at an equal key budget."""
import numpy as np
import pytest

from decode_attention_13_b200 import synth
from oracle import allocation, attention, quantize, rope


def _coded(seed, T, g_q, kb, vb, pairing=rope.HALF, dtype=np.float16, theta=1e4):
    hd = synth.head(seed, T=T, d=128, theta=theta, g_q=g_q, pairing=pairing, dtype=dtype)
    bits = allocation.greedy_bits(allocation.block_energy(hd["k"], pairing), kb, 128)
    kg = quantize.quantize_keys(hd["k"], bits, pairing)
    vg = quantize.quantize_values(hd["v"], vb)
    return hd, bits, kg, vg


@pytest.mark.parametrize("pairing", [rope.HALF, rope.INTERLEAVED])
def test_two_routes_agree(pairing):
    hd, bits, kg, vg = _coded((21,), 257, 4, 3, 3, pairing)
    a = attention.decode_rotated(hd["q"], kg, vg)
    b = attention.decode_dequantised(hd["q"], kg, vg)
    assert np.max(np.abs(a - b)) < 1e-12 * max(1.0, np.max(np.abs(a)))


def test_single_token_returns_its_value():
    hd, bits, kg, vg = _coded((22,), 1, 2, 2, 2)
    out = attention.decode_rotated(hd["q"], kg, vg)
    vhat = quantize.dequantize_values(vg)
    assert np.allclose(out, np.repeat(vhat[:1], 2, axis=0), atol=1e-12)


def test_equal_logits_average_values():
    hd, bits, kg, vg = _coded((23,), 50, 1, 3, 3)
    out = attention.decode_rotated(np.zeros((1, 128)), kg, vg)
    vhat = quantize.dequantize_values(vg)
    assert np.allclose(out[0], vhat.mean(axis=0), atol=1e-12)


def test_high_rate_approaches_exact_attention():
    hd = synth.head((24,), T=200, d=128, theta=1e4, g_q=2, dtype=np.float64)
    bits = allocation.greedy_bits(allocation.block_energy(hd["k"]), 7, 128)
    kg = quantize.quantize_keys(hd["k"], bits, rope.HALF)
    vg = quantize.quantize_values(hd["v"], 8)
    a = attention.decode_rotated(hd["q"], kg, vg)
    ex = attention.attention_exact(hd["q"], hd["k"], hd["v"])
    assert np.linalg.norm(a - ex) / np.linalg.norm(ex) < 0.02


@pytest.mark.parametrize("kb", [2, 3])
def test_block_gtq_logit_mae_not_above_uniform(kb):
    # K-only quantization at an equal key budget on synthetic heads
    ratios = []
    for s in range(6):
        hd = synth.head((30, s), T=512, d=128, theta=1e4, g_q=4, dtype=np.float16)
        bits = allocation.greedy_bits(allocation.block_energy(hd["k"]), kb, 128)
        kh_b = quantize.dequantize_keys(quantize.quantize_keys(hd["k"], bits, rope.HALF), 128, 512)
        kh_u = quantize.dequantize_keys(quantize.quantize_keys_uniform(hd["k"], kb, rope.HALF), 128, 512)
        mae_b = attention.logit_mae(hd["q"], hd["k"], kh_b)
        mae_u = attention.logit_mae(hd["q"], hd["k"], kh_u)
        assert mae_b <= mae_u
        ratios.append(mae_b / mae_u)
    print("Block-GTQ / uniform logit MAE at K%d:" % kb, np.round(ratios, 3))


def test_general_reduces_to_rotated_without_window():
    hd, bits, kg, vg = _coded((25,), 300, 4, 3, 3)
    a = attention.decode_general(hd["q"], kg, values=vg)
    b = attention.decode_rotated(hd["q"], kg, vg)
    assert np.max(np.abs(a - b)) < 1e-12 * max(1.0, np.max(np.abs(b)))
    c = attention.decode_general(hd["q"], kg, values=vg, k_recent=np.zeros((0, 128)),
                                 v_recent=np.zeros((0, 128)))
    assert np.max(np.abs(c - b)) < 1e-12 * max(1.0, np.max(np.abs(b)))


def test_key_only_matches_textbook_attention_on_dequantised_keys():
    # second route: rebuild k_hat in the original basis, textbook softmax with exact V
    hd, bits, kg, vg = _coded((26,), 333, 3, 3, 3)
    a = attention.decode_general(hd["q"], kg, v_fp16=hd["v"])
    k_hat = quantize.dequantize_keys(kg, 128, 333)
    q = hd["q"].astype(np.float64)
    s = q @ k_hat.T / np.sqrt(128)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    b = p @ hd["v"].astype(np.float64)
    assert np.max(np.abs(a - b)) < 1e-12 * max(1.0, np.max(np.abs(b)))


def test_window_holding_every_token_is_exact_attention():
    hd = synth.head((27,), T=200, d=128, theta=1e4, g_q=4, dtype=np.float16)
    empty = quantize.quantize_keys(hd["k"][:0], np.full(64, 3), rope.HALF)
    a = attention.decode_general(hd["q"], empty, v_fp16=hd["v"][:0], k_recent=hd["k"],
                                 v_recent=hd["v"])
    ex = attention.attention_exact(hd["q"], hd["k"], hd["v"])
    assert np.max(np.abs(a - ex)) < 1e-12 * max(1.0, np.max(np.abs(ex)))


def test_window_after_coded_tokens_is_one_softmax():
    # coded prefix + fp16 window == textbook attention over [k_hat ; k_window]
    hd, bits, kg_all, vg_all = _coded((28,), 260, 2, 3, 3)
    T = 200
    kg = quantize.quantize_keys(hd["k"][:T], bits, rope.HALF)
    vg = quantize.quantize_values(hd["v"][:T], 3)
    a = attention.decode_general(hd["q"], kg, values=vg, k_recent=hd["k"][T:],
                                 v_recent=hd["v"][T:])
    k_all = np.concatenate([quantize.dequantize_keys(kg, 128, T), hd["k"][T:].astype(np.float64)])
    v_all = np.concatenate([quantize.dequantize_values(vg), hd["v"][T:].astype(np.float64)])
    q = hd["q"].astype(np.float64)
    s = q @ k_all.T / np.sqrt(128)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    b = p @ v_all
    assert np.max(np.abs(a - b)) < 1e-12 * max(1.0, np.max(np.abs(b)))
