"""GPU parity of libgtq against the fp64 oracle, through the C ABI.

Tolerances (the construction's match criteria):
  * allocations: bit-exact;
  * energies: relative 1e-12 (fp64 sums in a different order);
  * codes: bit-exact except at most 1e-4 of them one level off -- the GPU takes
    the threshold decision in fp32 on an fp32 rotation, the oracle rounds its
    fp64 value to fp32 before the same decision, so only values within fp32
    rounding of a threshold can differ;
  * stored fp16 norms: bit-exact except at most 1e-4 of them one ulp off (fp64
    sums in another order);
  * decode outputs: relative L2 <= 2e-3 on identical packed inputs (the oracle's
    codes written into the layout by tests/layout.py).
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import decode_attention_13_b200 as gtq  # noqa: E402
from decode_attention_13_b200 import synth  # noqa: E402
from oracle import allocation, attention, lloyd_max, quantize  # noqa: E402
from tests import layout  # noqa: E402

pytestmark = pytest.mark.gpu

CODE_FLIP_MAX = 1e-4
NORM_ULP_MAX = 1e-4
DECODE_REL_L2 = 2e-3


def rel_l2(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


class Case:
    """One layer run through the library, with the oracle's view of every head."""

    def __init__(self, B, hkv, gq, T, kb, vb, pairing=0, dtype="fp16", seed=0, theta=1e4,
                 cap=None, decay=None):
        self.B, self.hkv, self.gq, self.T, self.kb, self.vb = B, hkv, gq, T, kb, vb
        self.pairing = pairing
        npdt = np.float16 if dtype == "fp16" else np.float32
        self.lay = synth.layer((seed,), B, hkv, gq, T, theta=theta, pairing=pairing,
                               dtype=npdt, decay=decay)
        self.cap = cap or T
        k = torch.zeros((B, hkv, self.cap, 128), dtype=torch.float16 if dtype == "fp16" else torch.float32)
        v = torch.zeros_like(k)
        k[:, :, :T] = torch.from_numpy(self.lay["k"])
        v[:, :, :T] = torch.from_numpy(self.lay["v"])
        self.k, self.v = k.cuda(), v.cuda()
        self.q = torch.from_numpy(self.lay["q"]).cuda()
        self.cfg = gtq.make_config(B, hkv * gq, hkv, kb, vb, self.cap, rope_pairing=pairing,
                                   in_dtype=gtq.DTYPE_FP16 if dtype == "fp16" else gtq.DTYPE_FP32)
        self.plan = gtq.gtq_alloc_bits(self.cfg, self.k, T)
        self.packed = torch.zeros(self.plan.packed_bytes, dtype=torch.uint8, device="cuda")

    def quantize(self, t0=0, n=None):
        gtq.gtq_quantize_pack(self.plan, self.k, self.v, t0, self.T - t0 if n is None else n,
                              self.packed)

    def decode(self, packed=None):
        out = torch.empty((self.B, self.hkv * self.gq, 128), dtype=torch.float32, device="cuda")
        gtq.gtq_decode_attn(self.plan, self.packed if packed is None else packed, self.T, self.q, out)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    def head_bytes(self, b, h, packed=None):
        p = (self.packed if packed is None else packed).cpu().numpy()
        per = self.plan.packed_bytes // (self.B * self.hkv)
        i = b * self.hkv + h
        return p[i * per:(i + 1) * per]

    # oracle side ----------------------------------------------------------
    def oracle_head(self, b, h):
        k = self.lay["k"][b, h]
        e = allocation.block_energy(k, self.pairing)
        bits = allocation.greedy_bits(e, self.kb, 128)
        kg = quantize.quantize_keys(k, bits, self.pairing)
        vg = quantize.quantize_values(self.lay["v"][b, h], self.vb)
        return e, bits, kg, vg


def compare_codes(case, b, h, kg, vg, bits):
    keys, vcodes, vnorm = layout.read_head(case.head_bytes(b, h), bits, case.kb, case.vb, case.T)
    by_w = {g.width: g for g in kg}
    flips = total = nflip = ntot = 0
    for (w, codes, n16) in keys:
        og = by_w[w]
        d = codes - og.codes
        assert np.all(np.abs(d) <= 1), "code off by more than one level"
        flips += int(np.count_nonzero(d))
        total += d.size
        nd = n16.view(np.uint16).astype(np.int64) - og.norm16.view(np.uint16).astype(np.int64)
        assert np.all(np.abs(nd) <= 1)
        nflip += int(np.count_nonzero(nd))
        ntot += nd.size
    d = vcodes - vg.codes
    assert np.all(np.abs(d) <= 1)
    flips += int(np.count_nonzero(d))
    total += d.size
    nd = vnorm.view(np.uint16).astype(np.int64) - vg.norm16.view(np.uint16).astype(np.int64)
    assert np.all(np.abs(nd) <= 1)
    nflip += int(np.count_nonzero(nd))
    ntot += nd.size
    assert flips <= CODE_FLIP_MAX * total, (flips, total)
    assert nflip <= NORM_ULP_MAX * ntot, (nflip, ntot)
    return flips, total


def check_case(case, check_decode=True, quantized=False):
    if not quantized:
        case.quantize()
    out_gpu_e2e = case.decode()
    bits_gpu = gtq.gtq_get_bits(case.plan)
    e_gpu = gtq.gtq_get_energy(case.plan)
    assert gtq.gtq_status(case.plan) == gtq.GTQ_OK
    oracle_packed = np.zeros(case.plan.packed_bytes, np.uint8)
    per = case.plan.packed_bytes // (case.B * case.hkv)
    n_tiles = per // layout.tile_bytes(case.kb, case.vb)
    ref_out = np.zeros((case.B, case.hkv * case.gq, 128))
    for b in range(case.B):
        for h in range(case.hkv):
            e, bits, kg, vg = case.oracle_head(b, h)
            assert np.allclose(e_gpu[b, h], e, rtol=1e-12, atol=0)
            assert np.array_equal(bits_gpu[b, h].astype(np.int64), bits), (b, h)
            compare_codes(case, b, h, kg, vg, bits)
            q = case.lay["q"][b, h * case.gq:(h + 1) * case.gq]
            ref_out[b, h * case.gq:(h + 1) * case.gq] = attention.decode_rotated(q, kg, vg)
            desc = sorted(kg, key=lambda g: -g.width)
            buf = layout.write_head(bits, [(g.width, g.codes, g.norm16) for g in desc],
                                    vg.codes, vg.norm16, case.kb, case.vb, n_tiles)
            i = b * case.hkv + h
            oracle_packed[i * per:(i + 1) * per] = buf
    if check_decode:
        out_same_codes = case.decode(torch.from_numpy(oracle_packed).cuda())
        assert rel_l2(out_same_codes, ref_out) <= DECODE_REL_L2
        assert rel_l2(out_gpu_e2e, ref_out) <= DECODE_REL_L2
    return ref_out


@pytest.mark.parametrize("B,hkv,gq,T,kb,vb,pairing,dtype", [
    (1, 1, 1, 1024, 3, 3, 0, "fp32"),       # the single-head fp32 correctness workload
    (2, 2, 4, 1000, 2, 2, 0, "fp16"),
    (1, 2, 8, 777, 3, 3, 1, "fp16"),
    (1, 1, 7, 129, 3, 2, 0, "fp16"),
    (1, 3, 2, 300, 4, 4, 0, "fp16"),
    (1, 1, 8, 200, 1, 1, 0, "fp16"),
    (1, 1, 8, 190, 8, 8, 1, "fp16"),
    (1, 1, 5, 257, 5, 3, 0, "fp32"),
    # wide tiles: fewer warp pairs per CTA, with enough tiles for two merge levels
    (1, 1, 8, 8192, 8, 8, 0, "fp16"),
    (2, 1, 4, 4000, 8, 6, 1, "fp16"),
    # groups of more than 8 query heads: several units (8 query heads each) per KV
    # head, the last one partial (9 = 8 + 1, 12 = 8 + 4), fp32 queries, and two
    # merge levels per unit
    (1, 1, 9, 333, 3, 2, 1, "fp16"),
    (2, 2, 12, 1500, 3, 3, 0, "fp32"),
    (1, 2, 16, 8192, 4, 4, 0, "fp16"),
    (1, 1, 32, 4100, 2, 2, 0, "fp16"),
])
def test_layer_parity(B, hkv, gq, T, kb, vb, pairing, dtype):
    check_case(Case(B, hkv, gq, T, kb, vb, pairing, dtype, seed=100 + T))


def test_many_heads_quantize_split():
    # 64 heads, fewer than three SMs each: the quantizer deals every head's tiles
    # to 2u key CTAs and u value CTAs (u = 2 here) that run in waves
    check_case(Case(16, 4, 2, 2560, 3, 2, seed=61))


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 128, 129])
def test_ragged_lengths(T):
    check_case(Case(1, 2, 4, T, 3, 3, seed=T))


def test_capacity_larger_than_T():
    check_case(Case(1, 1, 8, 150, 3, 3, cap=1000, seed=5))


def test_append_in_pieces():
    # one call for a prefix, a single-token append, then the rest: tokens are
    # written by different kernels (tensor-core tiles / CUDA-core edges); the
    # cache must still match the oracle, and other tokens' bytes are preserved
    c = Case(1, 2, 8, 700, 3, 3, seed=9)
    c.quantize(0, 333)
    c.quantize(333, 1)
    c.quantize(334, 700 - 334)
    torch.cuda.synchronize()
    check_case(c, quantized=True)


def test_zero_vectors():
    c = Case(1, 1, 4, 100, 3, 3, seed=3)
    c.k[:, :, 10] = 0
    c.v[:, :, 20] = 0
    c.lay["k"][:, :, 10] = 0
    c.lay["v"][:, :, 20] = 0
    c.plan = gtq.gtq_alloc_bits(c.cfg, c.k, c.T)
    check_case(c)


def test_norm_overflow_flagged():
    c = Case(1, 1, 1, 64, 2, 2, seed=4)
    c.v[0, 0, 5] = 60000.0           # |v| far above 65504
    c.quantize()
    torch.cuda.synchronize()
    assert gtq.gtq_status(c.plan) == gtq.GTQ_ERR_OVERFLOW
    assert gtq.gtq_status(c.plan) == gtq.GTQ_OK   # reading clears it


def _rebuild(c, k=None, v=None):
    """Replace the case's inputs (numpy fp16, [B, hkv, T, 128]) and re-plan."""
    if k is not None:
        c.lay["k"] = k
        c.k[:, :, :c.T] = torch.from_numpy(k).cuda()
    if v is not None:
        c.lay["v"] = v
        c.v[:, :, :c.T] = torch.from_numpy(v).cuda()
    c.plan = gtq.gtq_alloc_bits(c.cfg, c.k, c.T)


def test_zero_vectors_in_full_tiles():
    # zero key / value vectors inside 128-token tiles (tensor-core quantizer)
    c = Case(1, 2, 2, 300, 3, 3, seed=31)
    k, v = c.lay["k"].copy(), c.lay["v"].copy()
    k[:, :, [5, 140, 255]] = 0
    v[:, 1, [0, 129, 200]] = 0
    _rebuild(c, k, v)
    check_case(c)


def test_norm_overflow_in_full_tiles():
    c = Case(1, 1, 2, 256, 3, 3, seed=32)
    v = c.lay["v"].copy()
    v[0, 0, 140] = 30000.0           # |v| = 30000 sqrt(128), clamped to 65504
    k = c.lay["k"].copy()
    k[0, 0, 7] = 20000.0
    _rebuild(c, k, v)
    c.quantize()
    torch.cuda.synchronize()
    assert gtq.gtq_status(c.plan) == gtq.GTQ_ERR_OVERFLOW
    bits = gtq.gtq_get_bits(c.plan)[0, 0].astype(np.int64)
    _, obits, kg, vg = c.oracle_head(0, 0)
    assert np.array_equal(bits, obits)
    compare_codes(c, 0, 0, kg, vg, obits)


def test_subnormal_inputs():
    # values around 2^-20: most fp16 inputs are subnormal
    c = Case(1, 2, 2, 384, 3, 3, seed=33)
    k = (c.lay["k"].astype(np.float32) * 2.0 ** -20).astype(np.float16)
    v = (c.lay["v"].astype(np.float32) * 2.0 ** -20).astype(np.float16)
    _rebuild(c, k, v)
    check_case(c, check_decode=False)


def test_many_tiles_per_cta():
    # 32 heads: every quantizer CTA walks many 128-token tiles (pipeline phases)
    check_case(Case(4, 8, 1, 4096 + 77, 3, 3, seed=34))


@pytest.mark.parametrize("d", [4, 6, 8, 10])
@pytest.mark.parametrize("budget", [1, 2, 3, 4])
def test_greedy_from_energy_tiny_heads(d, budget):
    rng = np.random.default_rng(d * 7 + budget)
    E = rng.exponential(1.0, (3, 2, d // 2)) * np.exp(rng.uniform(-5, 5, (3, 2, d // 2)))
    cfg = gtq.make_config(3, 2, 2, budget, 2, 64, head_dim=d)
    plan = gtq.gtq_alloc_bits_from_energy(cfg, E)
    got = gtq.gtq_get_bits(plan)
    for b in range(3):
        for h in range(2):
            want = allocation.greedy_bits(E[b, h], budget, d)
            assert np.array_equal(got[b, h].astype(np.int64), want)


def test_greedy_equal_energies_uniform():
    for kb in (1, 2, 3, 5, 8):
        cfg = gtq.make_config(1, 1, 1, kb, 2, 64)
        plan = gtq.gtq_alloc_bits_from_energy(cfg, np.full((1, 1, 64), 0.25))
        assert np.all(gtq.gtq_get_bits(plan) == kb)


def test_greedy_ties_and_cap():
    cfg = gtq.make_config(1, 1, 1, 4, 2, 64, head_dim=16)
    E = np.array([[[1e12] + [1e-12] * 7]])
    plan = gtq.gtq_alloc_bits_from_energy(cfg, E)
    got = gtq.gtq_get_bits(plan)[0, 0].astype(np.int64)
    assert np.array_equal(got, allocation.greedy_bits(E[0, 0], 4, 16)) and got[0] == 8
    cfg = gtq.make_config(1, 1, 1, 3, 2, 64, head_dim=8)
    E = np.array([[[2.0, 2.0, 1.0, 1.0]]])
    plan = gtq.gtq_alloc_bits_from_energy(cfg, E)
    assert np.array_equal(gtq.gtq_get_bits(plan)[0, 0].astype(np.int64),
                          allocation.greedy_bits(E[0, 0], 3, 8))


def test_config0_as_stated():
    # the single-head correctness workload exactly as specified: d = 128,
    # T = 1024, theta = 1e4, one query at position T, decay a = 3 with two
    # outlier blocks x8, values N(0,1), K3V3, fp32 inputs, seed 0
    c = synth.CONFIGS[0]
    assert (c["T"], c["theta"], c["k_bits"], c["v_bits"], c["decay"], c["dtype"]) == \
        (1024, 1e4, 3, 3, 3.0, "fp32")
    hd = synth.head(0, T=c["T"], d=128, theta=c["theta"], g_q=1, decay=c["decay"],
                    dtype=np.float32)
    case = Case.__new__(Case)
    case.B, case.hkv, case.gq, case.T, case.kb, case.vb, case.pairing = 1, 1, 1, 1024, 3, 3, 0
    case.lay = {"k": hd["k"][None, None], "v": hd["v"][None, None], "q": hd["q"][None]}
    case.cap = case.T
    case.k = torch.from_numpy(case.lay["k"]).cuda()
    case.v = torch.from_numpy(case.lay["v"]).cuda()
    case.q = torch.from_numpy(case.lay["q"]).cuda()
    case.cfg = gtq.make_config(1, 1, 1, 3, 3, 1024, in_dtype=gtq.DTYPE_FP32)
    case.plan = gtq.gtq_alloc_bits(case.cfg, case.k, case.T)
    case.packed = torch.zeros(case.plan.packed_bytes, dtype=torch.uint8, device="cuda")
    ref = check_case(case)
    # the quantized decode stays close to unquantized attention on this head
    exact = attention.attention_exact(hd["q"], hd["k"], hd["v"])
    assert rel_l2(ref[0], exact) < 0.25


@pytest.mark.parametrize("pairing,dtype", [(0, "fp16"), (1, "fp16"), (0, "fp32")])
def test_append_under_frozen_allocation(pairing, dtype):
    # the serving loop: widths are chosen from a prefix of T_p tokens, the
    # prefix is quantized, then tokens are appended one or a few at a time with
    # those widths, and the decode covers every token written so far
    T_p, extra = 640, 16
    c = Case(1, 2, 4, T_p + extra, 3, 3, pairing=pairing, dtype=dtype, seed=61)
    c.plan = gtq.gtq_alloc_bits(c.cfg, c.k, T_p)            # energies of the prefix only
    gtq.gtq_quantize_pack(c.plan, c.k, c.v, 0, T_p, c.packed)
    bits_gpu = gtq.gtq_get_bits(c.plan)
    t = T_p
    for n in (1, 1, 2, 4, 8):                                 # 16 appended tokens
        gtq.gtq_quantize_pack(c.plan, c.k, c.v, t, n, c.packed)
        t += n
        c.T = t
        out = c.decode()                                      # same stream, no sync between
        ref = np.zeros_like(out, dtype=np.float64)
        for h in range(c.hkv):
            k = c.lay["k"][0, h]
            bits = allocation.greedy_bits(allocation.block_energy(k[:T_p], pairing), 3, 128)
            assert np.array_equal(bits_gpu[0, h].astype(np.int64), bits)
            kg = quantize.quantize_keys(k[:t], bits, pairing)   # all tokens, prefix widths
            vg = quantize.quantize_values(c.lay["v"][0, h][:t], 3)
            compare_codes(c, 0, h, kg, vg, bits)
            q = c.lay["q"][0, h * c.gq:(h + 1) * c.gq]
            ref[0, h * c.gq:(h + 1) * c.gq] = attention.decode_rotated(q, kg, vg)
        assert rel_l2(out, ref) <= DECODE_REL_L2, t
    assert gtq.gtq_status(c.plan) == gtq.GTQ_OK
