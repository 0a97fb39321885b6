"""Parity at the full workload sizes, in the launch configuration bench.py times.

For each of the four fp16 workloads (one layer of it: the library's unit), the
library builds the packed cache of the whole layer (energy, greedy allocation,
quantize-pack) and decodes it with one gtq_decode_attn call, exactly as the
benchmark does.  The oracle then checks:
  * every KV head: its block energies (fp64, rtol 1e-12) and its bit
    allocation (exact, the oracle's greedy on fp64 energies);
  * four KV heads (first, last, and two others; in the batched workload two of
    them come from different sequences): the codes and norms of 4096 sampled
    tokens plus the first and last tile (codes within one level, <= 1e-4 of
    them off; norms within one fp16 ulp, <= 1e-4 of them off), and the
    attention output of their query heads, decoded by the oracle from the codes
    read back out of the library's packed cache (identical packed inputs),
    within 2e-3 relative L2.

Energies for the allocation check are vectorised fp64 sums (pairwise order);
where the greedy decision is close enough to a tie that a relative change of
1e-12 in the energies changes it, the head's energies are recomputed with the
oracle's correctly rounded sums (math.fsum) before the comparison.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import decode_attention_13_b200 as gtq  # noqa: E402
from decode_attention_13_b200 import synth  # noqa: E402
from oracle import allocation, attention, quantize  # noqa: E402

from tests import layout  # noqa: E402

pytestmark = pytest.mark.gpu

CODE_FLIP_MAX = 1e-4
NORM_ULP_MAX = 1e-4
DECODE_REL_L2 = 2e-3
SAMPLE_TOKENS = 4096


def _rel_l2(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


def _energy_vec(k_head):
    """E_i of one head from its fp16 keys [T, 128] (HALF pairing), fp64."""
    kk = k_head.astype(np.float64)
    sq = np.sum(kk * kk, axis=0)
    return (sq[:64] + sq[64:]) / kk.shape[0]


def _oracle_bits(k_head, kb):
    e = _energy_vec(k_head)
    bits = allocation.greedy_bits(e, kb, 128)
    for f in (1 + 1e-12, 1 - 1e-12):
        rng = np.random.default_rng(int(f * 1e6))
        alt = allocation.greedy_bits(e * (1 + (f - 1) * rng.uniform(-1, 1, e.shape)), kb, 128)
        if not np.array_equal(alt, bits):        # near-tie: use the exact sums
            e = allocation.block_energy(k_head, 0)
            return e, allocation.greedy_bits(e, kb, 128)
    return e, bits


def _check_head_codes(head_bytes, bits, kb, vb, T, k_np, v_np, seed):
    keys, vcodes, vnorm = layout.read_head(head_bytes, bits, kb, vb, T)
    rng = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([np.arange(min(64, T)), np.arange(max(0, T - 64), T),
                                    rng.choice(T, min(T, SAMPLE_TOKENS), replace=False)]))
    kg = quantize.quantize_keys(k_np[idx], bits, 0)
    vg = quantize.quantize_values(v_np[idx], vb)
    by_w = {g.width: g for g in kg}
    flips = total = nflip = ntot = 0
    pairs = [(codes[idx], n16[idx], by_w[w].codes, by_w[w].norm16) for (w, codes, n16) in keys]
    pairs.append((vcodes[idx], vnorm[idx], vg.codes, vg.norm16))
    for c_got, n_got, c_ref, n_ref in pairs:
        d = c_got - c_ref
        assert np.all(np.abs(d) <= 1)
        flips += int(np.count_nonzero(d))
        total += d.size
        nd = n_got.view(np.uint16).astype(np.int64) - n_ref.view(np.uint16).astype(np.int64)
        assert np.all(np.abs(nd) <= 1)
        nflip += int(np.count_nonzero(nd))
        ntot += nd.size
    assert flips <= CODE_FLIP_MAX * total, (flips, total)
    assert nflip <= NORM_ULP_MAX * ntot, (nflip, ntot)
    # the library's own codes as the oracle's decode input
    coords = {g.width: g.coords for g in kg}
    ok = [quantize.CodedGroup(w, coords[w], c, n, n.astype(np.float64), False)
          for (w, c, n) in keys]
    ov = quantize.CodedGroup(vb, vg.coords, vcodes, vnorm, vnorm.astype(np.float64), False)
    return ok, ov


def _sampled_heads(B, hkv):
    heads = {(0, 0), (B - 1, hkv - 1)}
    if B > 1:
        heads |= {(B // 2, hkv // 2), (1, hkv - 1)}
    else:
        heads |= {(0, hkv // 2), (0, max(0, hkv // 2 - 1))}
    return sorted(heads)


@pytest.mark.parametrize("config", [1, 2, 3, 4])
def test_full_size_layer(config):
    c = synth.CONFIGS[config]
    B, hq, hkv, T, kb, vb = c["B"], c["h_q"], c["h_kv"], c["T"], c["k_bits"], c["v_bits"]
    gq = hq // hkv
    k, v, q = synth.layer_torch((config, 0, 0), B, hkv, gq, T, theta=c["theta"],
                                decay=c["decay"], device="cuda")
    cfg = gtq.make_config(B, hq, hkv, kb, vb, T)
    plan = gtq.gtq_alloc_bits(cfg, k, T)
    packed = torch.empty(plan.packed_bytes, dtype=torch.uint8, device="cuda")
    gtq.gtq_quantize_pack(plan, k, v, 0, T, packed)
    out = torch.empty((B, hq, 128), dtype=torch.float32, device="cuda")
    gtq.gtq_decode_attn(plan, packed, T, q, out)
    torch.cuda.synchronize()
    assert gtq.gtq_status(plan) == gtq.GTQ_OK
    bits_gpu = gtq.gtq_get_bits(plan)
    e_gpu = gtq.gtq_get_energy(plan)

    # every head: energies and allocation
    for b in range(B):
        k_b = k[b].cpu().numpy()
        for h in range(hkv):
            e, bits = _oracle_bits(k_b[h], kb)
            assert np.allclose(e_gpu[b, h], e, rtol=1e-12, atol=0), (b, h)
            assert np.array_equal(bits_gpu[b, h].astype(np.int64), bits), (b, h)

    # sampled heads: codes, norms and the decode output on identical codes
    per = plan.packed_bytes // (B * hkv)
    out_np = out.cpu().numpy()
    for (b, h) in _sampled_heads(B, hkv):
        k_np = k[b, h].cpu().numpy()
        v_np = v[b, h].cpu().numpy()
        q_np = q[b, h * gq:(h + 1) * gq].float().cpu().numpy()
        bits = bits_gpu[b, h].astype(np.int64)
        head = packed[(b * hkv + h) * per:(b * hkv + h + 1) * per].cpu().numpy()
        ok, ov = _check_head_codes(head, bits, kb, vb, T, k_np, v_np, config * 1000 + b * 10 + h)
        ref = attention.decode_rotated(q_np, ok, ov)
        assert _rel_l2(out_np[b, h * gq:(h + 1) * gq], ref) <= DECODE_REL_L2, (b, h)


def test_full_size_key_only_with_window():
    # the headline layer's shape (T = 131072, 16q/2kv) as a K-only plan (keys
    # coded at 3 bits, values read in fp16) with a 128-row fp16 window, decoded
    # in one gtq_decode_attn_full call as the bench's variants do; every head
    # checked: widths, sampled key codes and norms, and the output against the
    # oracle's decode of the library's own key codes, the fp16 values and the
    # window rows
    c = synth.CONFIGS[2]
    B, hq, hkv, T, kb, W = c["B"], c["h_q"], c["h_kv"], c["T"], c["k_bits"], 128
    gq = hq // hkv
    k, v, q = synth.layer_torch((2, 0, 0), B, hkv, gq, T, theta=c["theta"], decay=c["decay"],
                                device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(5)
    rk = torch.randn((B, hkv, W, 128), generator=gen, device="cuda", dtype=torch.float16)
    rv = torch.randn((B, hkv, W, 128), generator=gen, device="cuda", dtype=torch.float16)
    torch.cuda.synchronize()
    plan = gtq.gtq_alloc_bits(gtq.make_config(B, hq, hkv, kb, 0, T), k, T)
    packed = torch.empty(plan.packed_bytes, dtype=torch.uint8, device="cuda")
    gtq.gtq_quantize_pack(plan, k, None, 0, T, packed)
    out = torch.empty((B, hq, 128), dtype=torch.float32, device="cuda")
    gtq.gtq_decode_attn_full(plan, packed, T, q, out,
                             kv=gtq.fp16_kv(v=v, recent_k=rk, recent_v=rv))
    torch.cuda.synchronize()
    assert gtq.gtq_status(plan) == gtq.GTQ_OK
    bits_gpu = gtq.gtq_get_bits(plan)
    per = plan.packed_bytes // (B * hkv)
    out_np = out.cpu().numpy()
    for h in range(hkv):
        k_np = k[0, h].cpu().numpy()
        _, bits = _oracle_bits(k_np, kb)
        assert np.array_equal(bits_gpu[0, h].astype(np.int64), bits), h
        keys, vcodes, vnorm = layout.read_head(packed[h * per:(h + 1) * per].cpu().numpy(), bits,
                                               kb, 0, T)
        assert vcodes is None and vnorm is None
        rng = np.random.default_rng(77 + h)
        idx = np.unique(np.concatenate([np.arange(64), np.arange(T - 64, T),
                                        rng.choice(T, SAMPLE_TOKENS, replace=False)]))
        kg = quantize.quantize_keys(k_np[idx], bits, 0)
        by_w = {g.width: g for g in kg}
        flips = total = 0
        for (w, codes, n16) in keys:
            og = by_w[w]
            d = codes[idx] - og.codes
            assert np.all(np.abs(d) <= 1)
            flips += int(np.count_nonzero(d))
            total += d.size
            nd = (n16[idx].view(np.uint16).astype(np.int64)
                  - og.norm16.view(np.uint16).astype(np.int64))
            assert np.all(np.abs(nd) <= 1)
        assert flips <= CODE_FLIP_MAX * total, (flips, total)
        coords = {g.width: g.coords for g in kg}
        ok = [quantize.CodedGroup(w, coords[w], cc, n, n.astype(np.float64), False)
              for (w, cc, n) in keys]
        ref = attention.decode_general(q[0, h * gq:(h + 1) * gq].float().cpu().numpy(), ok,
                                       v_fp16=v[0, h].cpu().numpy(),
                                       k_recent=rk[0, h].cpu().numpy(),
                                       v_recent=rv[0, h].cpu().numpy())
        assert _rel_l2(out_np[0, h * gq:(h + 1) * gq], ref) <= DECODE_REL_L2, h
