"""GPU parity of the fp16 operands of decode (K-only plans and the fp16 window of
recent tokens) against the oracle's decode_general, through the C ABI.

K-only: a plan with v_bits = 0 codes the keys alone (the page's K-only
quantization, "RoPE-Aware Bit Allocation for KV-Cache Quantization", Abstract);
its codes and norms must match the oracle's (the criteria of the coded path),
and decode reads the values in fp16 from the caller's tensor.  Window: recent
tokens kept in fp16 beside the packed cache (the recent-key buffer the page's
headline result does without) are attended in the same softmax.

Decode tolerance: relative L2 <= 2e-3 on identical packed inputs, as for the
coded path (the kernels round P to fp16 for the tensor-core P.V).
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
DECODE_REL_L2 = 2e-3


def rel_l2(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


class Fp16Case:
    """B sequences of T packed tokens (lens[b] of them valid) plus W window rows
    (wlens[b] valid), all drawn as one synthetic layer of T + W tokens: the
    window holds the tokens after the packed ones."""

    def __init__(self, B, hkv, gq, T, kb, vb, W=0, lens=None, wlens=None, pairing=0, seed=0,
                 poison=True):
        self.B, self.hkv, self.gq, self.T, self.kb, self.vb, self.W = B, hkv, gq, T, kb, vb, W
        self.pairing = pairing
        lay = synth.layer((seed,), B, hkv, gq, T + W, theta=1e4, pairing=pairing)
        self.k_all, self.v_all, self.qn = lay["k"], lay["v"], lay["q"]
        self.lens = list(lens) if lens is not None else [T] * B
        self.wlens = list(wlens) if wlens is not None else [W] * B
        k = torch.from_numpy(np.ascontiguousarray(self.k_all[:, :, :T]))
        v = torch.from_numpy(np.ascontiguousarray(self.v_all[:, :, :T]))
        if poison:  # rows past a sequence's length hold garbage the kernels must not use
            for b in range(B):
                v[b, :, self.lens[b]:] = float("nan")
        self.k, self.v = k.cuda(), v.cuda()
        self.q = torch.from_numpy(self.qn).cuda()
        self.rk = torch.from_numpy(np.ascontiguousarray(self.k_all[:, :, T:])).cuda()
        self.rv = torch.from_numpy(np.ascontiguousarray(self.v_all[:, :, T:])).cuda()
        if poison and W:
            for b in range(B):
                self.rk[b, :, self.wlens[b]:] = float("nan")
                self.rv[b, :, self.wlens[b]:] = float("nan")
        self.seq_lens = torch.tensor(self.lens, dtype=torch.int32, device="cuda")
        self.rlens = torch.tensor(self.wlens, dtype=torch.int32, device="cuda")
        self.layout = gtq.seq_layout(self.seq_lens)
        self.cfg = gtq.make_config(B, hkv * gq, hkv, kb, vb, T, rope_pairing=pairing)
        # energies over each sequence's own tokens (NaN rows are values, not keys)
        self.plan = gtq.gtq_alloc_bits_ex(self.cfg, self.k, T, layout=self.layout)
        self.packed = torch.zeros(self.plan.packed_bytes, dtype=torch.uint8, device="cuda")

    def quantize(self):
        gtq.gtq_quantize_pack_ex(self.plan, self.k, None if self.vb == 0 else self.v, 0, self.T,
                                 self.packed, layout=self.layout)

    def kv(self):
        return gtq.fp16_kv(v=self.v if self.vb == 0 else None,
                           recent_k=self.rk if self.W else None,
                           recent_v=self.rv if self.W else None,
                           recent_lens=self.rlens if self.W else None)

    def decode(self, packed=None):
        out = torch.full((self.B, self.hkv * self.gq, 128), float("nan"), dtype=torch.float32,
                         device="cuda")
        kv = self.kv()
        gtq.gtq_decode_attn_full(self.plan, self.packed if packed is None else packed, self.T,
                                 self.q, out, layout=self.layout, kv=kv)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    def per_head(self):
        return self.plan.packed_bytes // (self.B * self.hkv)


def check(case, check_codes=True):
    case.quantize()
    out_e2e = case.decode()
    assert gtq.gtq_status(case.plan) == gtq.GTQ_OK
    bits_gpu = gtq.gtq_get_bits(case.plan)
    per = case.per_head()
    n_tiles = per // layout.tile_bytes(case.kb, case.vb)
    packed_np = case.packed.cpu().numpy()
    oracle_packed = np.zeros(case.plan.packed_bytes, np.uint8)
    ref = np.zeros((case.B, case.hkv * case.gq, 128))
    for b in range(case.B):
        L, Wb = case.lens[b], case.wlens[b]
        for h in range(case.hkv):
            i = b * case.hkv + h
            q = case.qn[b, h * case.gq:(h + 1) * case.gq]
            kr = case.k_all[b, h, case.T:case.T + Wb] if Wb else None
            vr = case.v_all[b, h, case.T:case.T + Wb] if Wb else None
            if L == 0:
                if Wb:  # the window alone: plain attention over its fp16 rows
                    s = q.astype(np.float64) @ kr.astype(np.float64).T / np.sqrt(128)
                    p = np.exp(s - s.max(axis=1, keepdims=True))
                    ref[b, h * case.gq:(h + 1) * case.gq] = (p / p.sum(axis=1, keepdims=True)) @ vr
                continue    # nothing at all: a zero output
            k = case.k_all[b, h, :L]
            bits = allocation.greedy_bits(allocation.block_energy(k, case.pairing), case.kb, 128)
            assert np.array_equal(bits_gpu[b, h].astype(np.int64), bits), (b, h)
            kg = quantize.quantize_keys(k, bits, case.pairing)
            vg = quantize.quantize_values(case.v_all[b, h, :L], case.vb) if case.vb else None
            desc = sorted(kg, key=lambda g: -g.width)
            if check_codes:
                keys, vcodes, vnorm = layout.read_head(packed_np[i * per:(i + 1) * per], bits,
                                                       case.kb, case.vb, L)
                if case.vb == 0:
                    assert vcodes is None and vnorm is None
                flips = total = 0
                for (w, codes, n16), og in zip(keys, desc):
                    assert w == og.width
                    d = codes - og.codes
                    assert np.all(np.abs(d) <= 1)
                    flips += int(np.count_nonzero(d))
                    total += d.size
                    nd = n16.view(np.uint16).astype(np.int64) - og.norm16.view(np.uint16).astype(np.int64)
                    assert np.all(np.abs(nd) <= 1)
                assert flips <= CODE_FLIP_MAX * total + 1, (flips, total)
            buf = layout.write_head(bits, [(g.width, g.codes, g.norm16) for g in desc],
                                    None if vg is None else vg.codes,
                                    None if vg is None else vg.norm16, case.kb, case.vb, n_tiles)
            oracle_packed[i * per:(i + 1) * per] = buf
            ref[b, h * case.gq:(h + 1) * case.gq] = attention.decode_general(
                q, kg, values=vg, v_fp16=None if vg is not None else case.v_all[b, h, :L],
                k_recent=kr, v_recent=vr)
    out_same = case.decode(torch.from_numpy(oracle_packed).cuda())
    assert np.all(np.isfinite(out_same)) and np.all(np.isfinite(out_e2e))
    assert rel_l2(out_same, ref) <= DECODE_REL_L2, rel_l2(out_same, ref)
    assert rel_l2(out_e2e, ref) <= DECODE_REL_L2, rel_l2(out_e2e, ref)
    return ref


@pytest.mark.parametrize("B,hkv,gq,T,kb,pairing", [
    (2, 2, 4, 300, 3, 0),
    (1, 1, 8, 1000, 2, 1),
    (1, 2, 7, 129, 4, 0),
    (1, 1, 1, 64, 3, 0),
    (1, 1, 8, 8192, 3, 0),     # several splits and both merge levels
    (1, 2, 12, 900, 3, 0),     # a group of 12 query heads: units of 8 and 4
])
def test_key_only_parity(B, hkv, gq, T, kb, pairing):
    check(Fp16Case(B, hkv, gq, T, kb, 0, pairing=pairing, seed=400 + T))


def test_key_only_many_heads():
    # 52 heads, fewer than three SMs each: K-only plans deal every head's key
    # tiles to several CTAs that run in waves
    check(Fp16Case(13, 4, 2, 1700, 3, 0, seed=63))


def test_key_only_ragged_sequences():
    # rows past each length are NaN in the caller's value tensor; an empty sequence
    check(Fp16Case(3, 2, 4, 700, 3, 0, lens=[700, 65, 0], seed=7))


@pytest.mark.parametrize("vb", [0, 3])
def test_window_parity(vb):
    check(Fp16Case(2, 2, 4, 500, 3, vb, W=37, wlens=[37, 5], seed=11 + vb))


@pytest.mark.parametrize("vb", [0, 2])
def test_window_with_many_splits(vb):
    check(Fp16Case(1, 2, 8, 6000, 3, vb, W=300, seed=21 + vb))


@pytest.mark.parametrize("vb", [0, 3])
def test_window_with_large_query_groups(vb):
    # 16 and 20 query heads per KV head with a window, ragged packed and window lengths
    check(Fp16Case(2, 1, 16, 700, 3, vb, W=40, lens=[700, 130], wlens=[40, 9], seed=41 + vb))
    check(Fp16Case(1, 2, 20, 2100, 2, vb, W=70, seed=43 + vb))


@pytest.mark.parametrize("vb", [0, 3])
def test_window_on_every_split_of_many_units(vb):
    # 16 decode units (4 x 4 KV heads; 2 x 4 KV heads x 2 query slices): 10
    # splits each, and windows long enough (>= 10 blocks of 32 rows) that every
    # split attends window rows, filling every window partial slot of a unit
    check(Fp16Case(4, 4, 4, 1000, 3, vb, W=400, seed=51 + vb))
    check(Fp16Case(2, 4, 12, 900, 2, vb, W=333, wlens=[333, 100], seed=53 + vb))


def test_window_alone_is_plain_attention():
    # packed part empty in one sequence, window empty in another, both empty in a third
    check(Fp16Case(3, 1, 4, 200, 3, 3, W=50, lens=[0, 200, 0], wlens=[50, 0, 0], seed=31))


def test_argument_checks():
    c = Fp16Case(1, 1, 4, 128, 3, 0, W=8, seed=41, poison=False)
    c.quantize()
    out = torch.empty((1, 4, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(gtq.GtqError) as e:     # K-only plans need their fp16 values
        gtq.gtq_decode_attn_ex(c.plan, c.packed, c.T, c.q, out)
    assert e.value.code == gtq.GTQ_ERR_INVALID
    kv = c.kv()
    kv.recent_len = 2000                        # above the window bound
    with pytest.raises(gtq.GtqError):
        gtq.gtq_decode_attn_full(c.plan, c.packed, c.T, c.q, out, kv=kv)
    kv = c.kv()
    kv.v_strides[3] = 2
    with pytest.raises(gtq.GtqError):
        gtq.gtq_decode_attn_full(c.plan, c.packed, c.T, c.q, out, kv=kv)
    with pytest.raises(gtq.GtqError):           # K-only plans take no values to code
        gtq.gtq_quantize_pack(c.plan, c.k, c.v, 0, c.T, c.packed)
    coded = Fp16Case(1, 1, 4, 128, 3, 3, seed=42, poison=False)
    coded.quantize()
    with pytest.raises(gtq.GtqError):           # coded plans take no fp16 values
        gtq.gtq_decode_attn_full(coded.plan, coded.packed, coded.T, coded.q, out,
                                 kv=gtq.fp16_kv(v=coded.v))


def test_key_only_appends_with_window_and_fp32_queries():
    # K-only plan: widths from a prefix, tokens appended 1, 2 and 4 at a time
    # (the small-M path), each append followed by a decode on the same stream
    # with no sync in between; fp32 queries and a window of 24 fp16 rows
    T_p, W = 600, 24
    lay = synth.layer((71,), 1, 2, 4, T_p + 7 + W, theta=1e4)
    k_all, v_all = lay["k"], lay["v"]
    T = T_p + 7
    k = torch.from_numpy(np.ascontiguousarray(k_all[:, :, :T])).cuda()
    v = torch.from_numpy(np.ascontiguousarray(v_all[:, :, :T])).cuda()
    rk = torch.from_numpy(np.ascontiguousarray(k_all[:, :, T:])).cuda()
    rv = torch.from_numpy(np.ascontiguousarray(v_all[:, :, T:])).cuda()
    q32 = torch.from_numpy(lay["q"].astype(np.float32)).cuda()
    cfg = gtq.make_config(1, 8, 2, 3, 0, T)
    plan = gtq.gtq_alloc_bits(cfg, k, T_p)
    packed = torch.zeros(plan.packed_bytes, dtype=torch.uint8, device="cuda")
    gtq.gtq_quantize_pack(plan, k, None, 0, T_p, packed)
    kv = gtq.fp16_kv(v=v, recent_k=rk, recent_v=rv)
    t = T_p
    for n in (1, 2, 4):
        gtq.gtq_quantize_pack(plan, k, None, t, n, packed)
        t += n
        out = torch.empty((1, 8, 128), dtype=torch.float32, device="cuda")
        gtq.gtq_decode_attn_full(plan, packed, t, q32, out, kv=kv)
        torch.cuda.synchronize()
        ref = np.zeros((1, 8, 128))
        for h in range(2):
            bits = allocation.greedy_bits(allocation.block_energy(k_all[0, h, :T_p], 0), 3, 128)
            kg = quantize.quantize_keys(k_all[0, h, :t], bits, 0)
            ref[0, 4 * h:4 * h + 4] = attention.decode_general(
                lay["q"][0, 4 * h:4 * h + 4].astype(np.float32), kg, v_fp16=v_all[0, h, :t],
                k_recent=k_all[0, h, T:], v_recent=v_all[0, h, T:])
        assert rel_l2(out.cpu().numpy(), ref) <= DECODE_REL_L2, t
    assert gtq.gtq_status(plan) == gtq.GTQ_OK


def test_key_only_paged_pool_with_mixed_lengths():
    # K-only keys in a paged pool (pages in reversed order), fp16 values read
    # by token from the caller's tensor, sequences of their own lengths
    B, hkv, gq, T = 3, 2, 4, 450
    lens = [450, 130, 1]
    lay = synth.layer((72,), B, hkv, gq, T, theta=1e4)
    k = torch.from_numpy(lay["k"]).cuda()
    v = torch.from_numpy(lay["v"]).cuda()
    q = torch.from_numpy(lay["q"]).cuda()
    n_tiles = (T + 63) // 64
    pages = B * n_tiles
    table = torch.arange(pages - 1, -1, -1, dtype=torch.int32, device="cuda").view(B, n_tiles)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    lay_ = gtq.seq_layout(seq, table)
    cfg = gtq.make_config(B, hkv * gq, hkv, 3, 0, T)
    plan = gtq.gtq_alloc_bits_ex(cfg, k, T, layout=gtq.seq_layout(seq))
    tb = gtq.gtq_layout_tile_bytes(3, 0)
    pool = torch.zeros(pages * hkv * tb, dtype=torch.uint8, device="cuda")
    gtq.gtq_quantize_pack_ex(plan, k, None, 0, T, pool, layout=lay_)
    out = torch.empty((B, hkv * gq, 128), dtype=torch.float32, device="cuda")
    gtq.gtq_decode_attn_full(plan, pool, T, q, out, layout=lay_, kv=gtq.fp16_kv(v=v))
    torch.cuda.synchronize()
    bits_gpu = gtq.gtq_get_bits(plan)
    ref = np.zeros((B, hkv * gq, 128))
    for b in range(B):
        for h in range(hkv):
            kk = lay["k"][b, h, :lens[b]]
            bits = allocation.greedy_bits(allocation.block_energy(kk, 0), 3, 128)
            assert np.array_equal(bits_gpu[b, h].astype(np.int64), bits), (b, h)
            kg = quantize.quantize_keys(kk, bits, 0)
            ref[b, h * gq:(h + 1) * gq] = attention.decode_general(
                lay["q"][b, h * gq:(h + 1) * gq], kg, v_fp16=lay["v"][b, h, :lens[b]])
    assert rel_l2(out.cpu().numpy(), ref) <= DECODE_REL_L2
    assert gtq.gtq_status(plan) == gtq.GTQ_OK
