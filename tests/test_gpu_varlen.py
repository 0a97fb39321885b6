"""Batches of sequences of their own lengths, in contiguous and paged caches.

Every sequence b of the batch holds len_b tokens: its energies are the mean
over its own tokens, its codes are written only below len_b, and its query
attends to exactly its len_b tokens.  With a block table the packed cache is a
pool of pages (one 64-token tile of every KV head of a sequence per page);
pages no sequence names stay untouched.  Checked against the oracle with the
usual tolerances (allocations exact, codes and norms within one step on at
most 1e-4 of them, outputs within 2e-3 relative L2)."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import decode_attention_13_b200 as gtq  # noqa: E402
from decode_attention_13_b200 import synth  # noqa: E402
from oracle import allocation, attention, quantize  # noqa: E402
from tests import layout  # noqa: E402
from tests.test_gpu_parity import CODE_FLIP_MAX, DECODE_REL_L2, NORM_ULP_MAX, rel_l2  # noqa: E402

pytestmark = pytest.mark.gpu


def _compare(head_bytes, bits, kb, vb, T, kg, vg):
    keys, vcodes, vnorm = layout.read_head(head_bytes, bits, kb, vb, T)
    by_w = {g.width: g for g in kg}
    flips = total = nflip = ntot = 0
    pairs = [(c, n, by_w[w].codes, by_w[w].norm16) for (w, c, n) in keys]
    pairs.append((vcodes, vnorm, vg.codes, vg.norm16))
    for c_got, n_got, c_ref, n_ref in pairs:
        d = c_got - c_ref
        assert np.all(np.abs(d) <= 1)
        flips += int(np.count_nonzero(d))
        total += d.size
        nd = n_got.view(np.uint16).astype(np.int64) - n_ref.view(np.uint16).astype(np.int64)
        assert np.all(np.abs(nd) <= 1)
        nflip += int(np.count_nonzero(nd))
        ntot += nd.size
    assert flips <= CODE_FLIP_MAX * max(total, 1) + 0.5, (flips, total)
    assert nflip <= NORM_ULP_MAX * max(ntot, 1) + 0.5, (nflip, ntot)


class Ragged:
    def __init__(self, lens, hkv=2, gq=4, kb=3, vb=3, cap=None, paged=False, seed=0):
        self.lens = list(lens)
        self.B, self.hkv, self.gq, self.kb, self.vb = len(lens), hkv, gq, kb, vb
        self.cap = cap or max(max(lens), 1)
        self.lay = synth.layer((seed,), self.B, hkv, gq, self.cap, theta=1e4)
        self.k = torch.from_numpy(self.lay["k"]).cuda()
        self.v = torch.from_numpy(self.lay["v"]).cuda()
        self.q = torch.from_numpy(self.lay["q"]).cuda()
        self.seq_lens = torch.tensor(self.lens, dtype=torch.int32, device="cuda")
        self.cfg = gtq.make_config(self.B, hkv * gq, hkv, kb, vb, self.cap)
        self.tb = layout.tile_bytes(kb, vb)
        self.tiles = (self.cap + 63) // 64
        self.table = None
        if paged:
            rng = np.random.default_rng(seed + 1)
            n_pages = self.B * self.tiles + 5                  # spare pages stay unused
            perm = rng.permutation(n_pages)[:self.B * self.tiles]
            self.table = torch.tensor(perm.reshape(self.B, self.tiles), dtype=torch.int32,
                                      device="cuda")
            self.pool_pages = n_pages
        self.layout = gtq.seq_layout(self.seq_lens, self.table)

    def build(self):
        self.plan = gtq.gtq_alloc_bits_ex(self.cfg, self.k, self.cap, self.layout)
        if self.table is None:
            nbytes = self.plan.packed_bytes
        else:
            nbytes = self.pool_pages * self.hkv * self.tb
        self.packed = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device="cuda")
        return self

    def head_bytes(self, b, h):
        p = self.packed.cpu().numpy()
        if self.table is None:
            per = self.plan.packed_bytes // (self.B * self.hkv)
            i = b * self.hkv + h
            return p[i * per:(i + 1) * per]
        return layout.gather_paged_head(p, self.table[b].cpu().numpy(), self.hkv, h,
                                        self.tiles, self.tb)

    def decode(self):
        out = torch.full((self.B, self.hkv * self.gq, 128), float("nan"), dtype=torch.float32,
                         device="cuda")
        gtq.gtq_decode_attn_ex(self.plan, self.packed, self.cap, self.q, out, self.layout)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    def check(self):
        out = self.decode()
        bits_gpu = gtq.gtq_get_bits(self.plan)
        e_gpu = gtq.gtq_get_energy(self.plan)
        assert gtq.gtq_status(self.plan) == gtq.GTQ_OK
        for b, L in enumerate(self.lens):
            for h in range(self.hkv):
                k = self.lay["k"][b, h, :L]
                e = allocation.block_energy(k, 0) if L else np.zeros(64)
                assert np.allclose(e_gpu[b, h], e, rtol=1e-12, atol=0), (b, h)
                bits = allocation.greedy_bits(e, self.kb, 128)
                assert np.array_equal(bits_gpu[b, h].astype(np.int64), bits), (b, h)
                qh = self.lay["q"][b, h * self.gq:(h + 1) * self.gq]
                got = out[b, h * self.gq:(h + 1) * self.gq]
                if L == 0:
                    assert np.all(got == 0.0)
                    continue
                kg = quantize.quantize_keys(k, bits, 0)
                vg = quantize.quantize_values(self.lay["v"][b, h, :L], self.vb)
                _compare(self.head_bytes(b, h), bits, self.kb, self.vb, L, kg, vg)
                ref = attention.decode_rotated(qh, kg, vg)
                assert rel_l2(got, ref) <= DECODE_REL_L2, (b, h, L)


@pytest.mark.parametrize("paged", [False, True])
def test_mixed_lengths(paged):
    r = Ragged([1, 130, 777, 1100, 64], cap=1100, paged=paged, seed=71).build()
    gtq.gtq_quantize_pack_ex(r.plan, r.k, r.v, 0, r.cap, r.packed, r.layout)
    r.check()
    if paged:   # pages that no sequence's length reaches, and spare pages, keep their bytes
        pool = r.packed.cpu().numpy().reshape(r.pool_pages, r.hkv * r.tb)
        used = set()
        tbl = r.table.cpu().numpy()
        for b, L in enumerate(r.lens):
            used |= set(int(x) for x in tbl[b, :(L + 63) // 64])
        for p in range(r.pool_pages):
            if p not in used:
                assert np.all(pool[p] == 0xA5), p


def test_empty_sequence_and_kv8():
    r = Ragged([0, 300, 65], hkv=1, gq=8, kb=2, vb=2, cap=320, seed=72).build()
    gtq.gtq_quantize_pack_ex(r.plan, r.k, r.v, 0, r.cap, r.packed, r.layout)
    r.check()


@pytest.mark.parametrize("paged", [False, True])
def test_batched_tail_appends(paged):
    # each sequence grows from its own prefix, one or a few tokens per call,
    # with the allocation frozen at the prefixes; decodes run in between
    final = [200, 645, 1000, 70]
    prefix = [f - 9 for f in final]
    r = Ragged(final, cap=1024, paged=paged, seed=73)
    r.seq_lens.copy_(torch.tensor(prefix, dtype=torch.int32))
    r.build()
    gtq.gtq_quantize_pack_ex(r.plan, r.k, r.v, 0, r.cap, r.packed, r.layout)
    bits_prefix = gtq.gtq_get_bits(r.plan)
    cur = list(prefix)
    for n in (1, 3, 5):
        cur = [c + n for c in cur]
        r.seq_lens.copy_(torch.tensor(cur, dtype=torch.int32))
        gtq.gtq_quantize_pack_ex(r.plan, r.k, r.v, gtq.GTQ_T0_TAIL, n, r.packed, r.layout)
    assert cur == final
    r.lens = final
    out = r.decode()
    for b, L in enumerate(final):
        for h in range(r.hkv):
            bits = allocation.greedy_bits(
                allocation.block_energy(r.lay["k"][b, h, :prefix[b]], 0), r.kb, 128)
            assert np.array_equal(bits_prefix[b, h].astype(np.int64), bits)
            kg = quantize.quantize_keys(r.lay["k"][b, h, :L], bits, 0)
            vg = quantize.quantize_values(r.lay["v"][b, h, :L], r.vb)
            _compare(r.head_bytes(b, h), bits, r.kb, r.vb, L, kg, vg)
            ref = attention.decode_rotated(r.lay["q"][b, h * r.gq:(h + 1) * r.gq], kg, vg)
            assert rel_l2(out[b, h * r.gq:(h + 1) * r.gq], ref) <= DECODE_REL_L2
    assert gtq.gtq_status(r.plan) == gtq.GTQ_OK
