"""Parity at the full workload sizes, in the launch configuration bench.py times.

For each of the four fp16 workloads (one layer of it: the library's unit), the
library builds the packed cache of the whole layer (energy, greedy allocation,
quantize-pack) and decodes it with one gtq_decode_attn call, exactly as the
benchmark does.  The oracle then checks one sampled KV head in full:
  * its block energies (fp64, rtol 1e-12) and bit allocation (exact);
  * the codes and norms of 4096 sampled tokens plus the first and last tile
    (codes within one level, <= 1e-4 of them off; norms within one fp16 ulp,
    <= 1e-4 of them off);
  * the attention output of its query heads, decoded by the oracle from the
    codes read back out of the library's packed cache (identical packed inputs),
    within 2e-3 relative L2.
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

    b, h = B - 1, hkv - 1                                  # the sampled head
    k_np = k[b, h].cpu().numpy()
    v_np = v[b, h].cpu().numpy()
    q_np = q[b, h * gq:(h + 1) * gq].float().cpu().numpy()
    e = allocation.block_energy(k_np, 0)
    assert np.allclose(e_gpu[b, h], e, rtol=1e-12, atol=0)
    bits = allocation.greedy_bits(e, kb, 128)
    assert np.array_equal(bits_gpu[b, h].astype(np.int64), bits)

    per = plan.packed_bytes // (B * hkv)
    head = packed[(b * hkv + h) * per:(b * hkv + h + 1) * per].cpu().numpy()
    keys, vcodes, vnorm = layout.read_head(head, bits, kb, vb, T)

    # codes and norms of sampled tokens
    rng = np.random.default_rng(config)
    idx = np.unique(np.concatenate([np.arange(64), np.arange(T - 64, T),
                                    rng.choice(T, SAMPLE_TOKENS, replace=False)]))
    kg = quantize.quantize_keys(k_np[idx], bits, 0)
    vg = quantize.quantize_values(v_np[idx], vb)
    by_w = {g.width: g for g in kg}
    flips = total = nflip = ntot = 0
    for (w, codes, n16) in keys:
        d = codes[idx] - by_w[w].codes
        assert np.all(np.abs(d) <= 1)
        flips += int(np.count_nonzero(d))
        total += d.size
        nd = n16[idx].view(np.uint16).astype(np.int64) - by_w[w].norm16.view(np.uint16).astype(np.int64)
        assert np.all(np.abs(nd) <= 1)
        nflip += int(np.count_nonzero(nd))
        ntot += nd.size
    d = vcodes[idx] - vg.codes
    assert np.all(np.abs(d) <= 1)
    flips += int(np.count_nonzero(d))
    total += d.size
    nd = vnorm[idx].view(np.uint16).astype(np.int64) - vg.norm16.view(np.uint16).astype(np.int64)
    assert np.all(np.abs(nd) <= 1)
    nflip += int(np.count_nonzero(nd))
    ntot += nd.size
    assert flips <= CODE_FLIP_MAX * total, (flips, total)
    assert nflip <= NORM_ULP_MAX * ntot, (nflip, ntot)

    # the whole head's attention output on the library's own codes
    oracle_keys = []
    for (w, codes, n16) in keys:
        g = by_w[w]
        oracle_keys.append(quantize.CodedGroup(w, g.coords, codes, n16, n16.astype(np.float64), False))
    oracle_values = quantize.CodedGroup(vb, vg.coords, vcodes, vnorm, vnorm.astype(np.float64), False)
    ref = attention.decode_rotated(q_np, oracle_keys, oracle_values)
    got = out[b, h * gq:(h + 1) * gq].cpu().numpy()
    assert _rel_l2(got, ref) <= DECODE_REL_L2
