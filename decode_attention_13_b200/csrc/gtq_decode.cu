// Fused GQA decode attention over the Block-GTQ packed cache ("RoPE-Aware Bit
// Allocation for KV-Cache Quantization", Abstract: decoding is served straight
// from the packed cache).  No fp16 K or V is materialised: codes become
// tensor-core operands in registers.  One launch per call (decode_kernel),
// grid = (units, splits), one CTA per SM, 2 * np consumer warps (np pairs) and
// one producer warp.  A unit is a KV head and up to 8 of its query heads (the
// MMA's N): groups of more than 8 query heads per KV head run as several units
// over the same cache (a second unit's reads of a tile mostly hit L2).
//   setup    before the grid-dependency wait: the constant lookup tables (bulk
//            copy; an L2 prefetch of the CTA's tiles there measured 8% slower
//            over a 36-layer step).  After it: the head metadata, the key
//            rotation blocks and the queries by bulk copy; q_rot = M_h q for
//            the unit's query heads, from each group's m x m block
//            only, times log2(e) / (sqrt(d) sqrt(m_g)); its fp16 hi / lo MMA
//            fragments.
//   loop     the producer deals 7/8 of a head's tiles statically and the rest
//            from a per-head counter (two at a time, the next grab in flight;
//            every tile by the counter when the CTAs outnumber the SMs),
//            and bulk-copies two adjacent 64-token tiles per stage into a ring;
//            the pair that owns a tile splits it, 32 tokens per warp.  Scores:
//            mma.m16n8k16 (m16n8k8 for a group's last half k-tile) with
//            A = codebook values of 16 tokens x 16 rotated coords (pair tables)
//            and B = q_rot, per key group, scaled by the group's fp16 norms;
//            the groups that hold most of the energy take hi + lo operands
//            (A_hi q_hi + A_hi q_lo + A_lo q_hi).  Online softmax in base 2.
//            P.V: mma with A = V codebook values (16 dims x 16 tokens) and
//            B = P^T (movmatrix transpose of the score fragment), in V's
//            rotated basis.
//   merge    the CTA's warps, then the splits: the last CTA of each group of
//            16 splits merges the group (and fetches R_V^T's fragments), the
//            last group merges the rest and writes o = R_V^T o_rot / l with
//            mma (fp16 hi / lo parts).  Tickets and the tile counter return to
//            0 for the next call.
// K-only plans (values kept in fp16, the page's K-only quantization, Abstract)
// take decode_kernel<0, *>: each stage also receives the tiles' fp16 value rows
// by a tensor copy (128-byte swizzle, so that the transposing ldmatrix that
// forms A = V^T is free of bank conflicts), P.V runs in the original basis and
// no R_V^T product follows.  An fp16 window of recent tokens (the recent-key
// buffer the page's method does without, Abstract) is attended, in the
// decode_kernel<*, true> instantiations, by the first splits during setup on
// the tensor cores, each into a partial of its own; the finishing CTA merges
// those and combines them with the cache's part by their softmax sums.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstddef>
#include <cstring>

#include "gtq_internal.h"

namespace gtq {
namespace {

// 7 pairs + the producer: at most 4 warps per SM sub-partition, so every warp
// may hold 128 registers (a 17th warp would cap them at 96)
constexpr int kPairs = 7;                     // consumer warp pairs (at most)
constexpr int kCWarps = 2 * kPairs;           // consumer warps (at most)
constexpr int kThreads = (kCWarps + 1) * 32;  // + the producer warp
constexpr int kMaxRing = 32;                  // stages
// A stage holds two adjacent tiles fetched by one bulk copy: the copy engine
// of an SM takes a roughly fixed time per copy, so 7 KB copies stream at about
// half the HBM bandwidth and 14 KB copies at nearly all of it (measured).
constexpr int kTPS = 2;                       // tiles per stage
constexpr int kSkip = -1;                     // stage tile slot without a tile
constexpr int kEnd = -2;                      // no tiles left for the pair
constexpr int kGrab = 2;                      // tiles per counter grab
constexpr int kStaticEighths = 7;             // share of a head's tiles dealt out statically
constexpr uint32_t kTabSharedAddr = 163840;   // shared address of the lookup tables
constexpr int kSmemBytes = (int)kTabSharedAddr + kDecodeImageBytes;
constexpr int kPackPrefix = 24576;            // rotation-pack bytes fetched with the metadata
constexpr int kPackArea = (int)((kRotPackBytes + 127) & ~size_t(127));
constexpr int kWoStride = kD + 4;                          // floats per (warp, head) row
constexpr int kWoBytes = kCWarps * 8 * kWoStride * 4;      // warps' o at the merge
constexpr int kRvFragBytes = 8 * 8 * 32 * 32;             // R_V^T fragments (fp16 hi + lo)
constexpr int kRvOff = (kWoBytes + 127) & ~127;
constexpr int kTailBytes = kRvOff + kRvFragBytes;
constexpr uint64_t kWaitNs = 2000000000ull;    // bound of one wait
static_assert(kTabSharedAddr % kDecTabAlign == 0, "table region alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct DecodeArgs {
  const uint8_t* packed;
  const HeadMeta* meta;
  const float* rotpack;    // [heads][kRotPackMaxWords]
  const void* q;           // [B][Hq][128] fp16 or fp32 (q_fp32)
  const uint4* rv_frag;    // R_V^T as mma A fragments: [m-tile][k-tile][lane] {hi, lo}
  float* out;              // [B][Hq][128]
  const uint4* dec_image;  // lookup tables (kDecodeImageBytes)
  float* partials;         // [heads][slot_total][8][kPartialStride]
  int slot_groups, slot_window, slot_total;  // PartialSlots of the plan
  unsigned* tickets;       // [heads][kTicketStride]
  int* status;
  const int32_t* seq_lens;     // [B] tokens per sequence, or null: all T
  const int32_t* block_table;  // [B][max_blocks] tile pages, or null: contiguous per head
  int64_t max_blocks;
  int q_fp32;
  int hkv, gq, nqs;  // KV heads per sequence, query heads per KV head, query slices
  int64_t T;
  int64_t n_tiles;    // capacity tiles per head (contiguous layout)
  int tile_bytes;
  int stride;         // bytes per stage (kTPS tiles)
  int kb;
  int ring;           // stages
  int np;             // consumer warp pairs
  int64_t static_per; // tiles [split * static_per, +static_per) are this CTA's; the rest
                      // (from splits * static_per on) go out through the tile counter
  // K-only plans
  int voff;           // bytes of a stage before its value rows (kTPS x 16 KB, swizzled)
  int v_loads;        // tensor copies per tile: 1 (5-D map) or 2 (4-D map, one per half)
  // fp16 window of recent tokens
  const __half* rk;
  const __half* rv;
  int64_t rs0, rs1, rs2;
  const int32_t* rlens;
  int rlen;           // rows per head, 0: no window
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, unsigned bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// the same with an L2 cache policy
__device__ __forceinline__ void bulk_copy_hint(void* dst, const void* src, unsigned bytes,
                                               uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// bring bytes into L2 (no effect on the values any load returns)
// tensor copies of value rows into shared memory (no cluster multicast)
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, int c4, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
      "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// the packed cache is streamed once per call: evicted first, so that it does
// not push the tables and metadata out of L2
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// bounded wait on an mbarrier phase; false after about two seconds.  try_wait
// without a suspend-time hint blocks for a short, hardware-chosen time and
// returns as soon as the phase completes; a hint long enough to matter here
// woke the waiting producer microseconds late and starved the tile pipeline.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned phase) {
  uint64_t t0 = 0;
  for (unsigned i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    if (ok) return true;
    if ((i & 63u) == 63u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0)
        t0 = now;
      else if (now - t0 > kWaitNs)
        return false;
    }
  }
}

// named barrier of the consumer warps (the producer warp never takes part)
__device__ __forceinline__ void consumers_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma1688(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// programmatic dependent launch: wait for / release the neighbouring grids
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

struct DecodeSmem {
  alignas(16) HeadMeta meta;
  uint4 qf[kMaxKt][32];        // per k-tile & lane: hi(slot A), hi(slot B), lo(A), lo(B)
  uint4 wqf[8][32];            // the window's q fragments (original basis): hi, hi, lo, lo
  alignas(16) float qa[8][kD];  // gathered queries [coordinate][head], then the merged o_rot
  alignas(16) float qb[8][kD];  // the raw queries (bulk copy), then q_rot (scaled)
  uint4 gdesc[kMaxGroups];      // W | split << 4 | k16 tiles << 8 | half k-tile << 16; key
                                // offset; first k-tile; -
  uint64_t tab_bar;             // lookup tables landed
  uint64_t meta_bar;            // metadata + rotation-pack prefix landed
  uint64_t pack_bar;            // rest of the rotation pack landed
  uint64_t done_bar;            // query rotation done: the pack's stages may be filled
  uint64_t rv_bar;              // R_V landed
  uint64_t full[kMaxRing];      // stage holds its tiles (or end markers)
  uint64_t empty[kMaxRing];     // stage released by the warps of both tile slots
  int2 stage_tile[kMaxRing];    // tile of each slot, kSkip or kEnd
  float wm[kCWarps][8], wl[kCWarps][8], wsc[kCWarps][8], hm[8], hl[8];
  int flag;
  int failed;
};
static_assert(offsetof(DecodeSmem, qf) % 16 == 0 && offsetof(DecodeSmem, meta) % 16 == 0 &&
                  offsetof(DecodeSmem, qa) % 16 == 0 && offsetof(DecodeSmem, qb) % 16 == 0 &&
                  offsetof(DecodeSmem, gdesc) % 16 == 0 && offsetof(DecodeSmem, full) % 8 == 0,
              "shared-memory alignment");
static_assert(sizeof(HeadMeta) % 16 == 0, "metadata is bulk-copied");

// ---------------------------------------------------------------------------
// Code -> fp16 lookups.  Every table address is "(base | field << k) + OFF",
// base = region | lane bits (b32: lane * 4, b16: (lane & 15) * 8, bss: none).
// ---------------------------------------------------------------------------

// bits [P, P + N) of the little-endian bit string x[], moved to bit S, masked, OR orv
template <int P, int N, int S>
__device__ __forceinline__ uint32_t fld(const uint32_t* x, uint32_t orv) {
  constexpr int wd = P >> 5, sh = P & 31;
  constexpr uint32_t mask = ((1u << N) - 1u) << S;
  uint32_t v;
  if constexpr (sh + N <= 32) {
    if constexpr (sh >= S) v = x[wd] >> (sh - S);
    else v = x[wd] << (S - sh);
  } else {
    static_assert(sh >= S, "field layout");
    v = __funnelshift_r(x[wd], x[wd + 1], sh - S);
  }
  return (v & mask) | orv;
}

template <uint32_t OFF>
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(OFF));
  return v;
}
template <uint32_t OFF>
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(addr), "n"(OFF));
  return v;
}

struct TabBase {
  uint32_t b32, b16, bss;
};

// hi|lo word (fp16 hi in the low half) of the code of width W >= 5 at bits [P, P + W)
template <int W, int P>
__device__ __forceinline__ uint32_t single_code(const uint32_t* x, const TabBase& tb) {
  if constexpr (W == 5 || W == 6)
    return lds32<kTabS32(W)>(fld<P, W, 7>(x, tb.b32));
  else
    return lds32<kTabSS + kSingleOff(W)>(fld<P, W, 2>(x, tb.bss));
}

// hi (and, if LO, lo) half2 of codes (2U, 2U + 1) of width W from the bit string x
template <int W, int U, bool LO>
__device__ __forceinline__ void code_pair(const uint32_t* x, const TabBase& tb, uint32_t& hi,
                                          uint32_t& lo) {
  if constexpr (W <= 4) {
    if constexpr (LO) {
      const uint2 v = lds64<kTabP16(W)>(fld<2 * U * W, 2 * W, 7>(x, tb.b16));
      hi = v.x;
      lo = v.y;
    } else if constexpr (W <= 3) {
      hi = lds32<kTabP32(W)>(fld<2 * U * W, 2 * W, 7>(x, tb.b32));
    } else {
      hi = lds32<kTabP16(W)>(fld<2 * U * W, 2 * W, 7>(x, tb.b16));
    }
  } else {
    const uint32_t e0 = single_code<W, 2 * U * W>(x, tb);
    const uint32_t e1 = single_code<W, (2 * U + 1) * W>(x, tb);
    hi = __byte_perm(e0, e1, 0x5410);
    if constexpr (LO) lo = __byte_perm(e0, e1, 0x7632);
  }
}

// The lane's W bytes of one slot (4 tokens x 2 codes) at byte offset off of
// the tile, realigned to bit 0 of x[] (x[1] holds bits 32.. for W > 4).
template <int W>
__device__ __forceinline__ void load_slot(const uint8_t* tile, int off, uint32_t (&x)[2]) {
  if constexpr (W == 1) {
    x[0] = tile[off];
  } else if constexpr (W == 2) {
    x[0] = *reinterpret_cast<const uint16_t*>(tile + off);
  } else if constexpr (W == 4) {
    x[0] = *reinterpret_cast<const uint32_t*>(tile + off);
  } else if constexpr (W == 8) {
    const uint2 v = *reinterpret_cast<const uint2*>(tile + off);
    x[0] = v.x;
    x[1] = v.y;
  } else {
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(tile + (off & ~3));
    const uint32_t sh = (uint32_t)(off & 3) << 3;
    const uint32_t w0 = wp[0], w1 = wp[1];
    x[0] = __funnelshift_r(w0, w1, sh);
    if constexpr (W > 4) x[1] = __funnelshift_r(w1, wp[2], sh);
  }
}

// Scores of one key group for this warp's 32 tokens.  The group's slots run in
// k-tiles of 8 (16 coords; this lane's slots are t and t + 4 of each, tokens
// g + 8u for u = 4 wh .. 4 wh + 3, i.e. W bytes of each slot's 2W-byte lane
// portion); a last run of at most 4 slots is a half k-tile (m16n8k8).  Slots
// past the group's run within a k-tile read unrelated bits; their q is zero.
// Lookups always fetch hi and lo parts; only the groups marked split multiply
// the lo parts (A_hi q_lo + A_lo q_hi), so one body per width serves both and
// the hot code stays small.
template <int W>
__device__ __forceinline__ void group_scores(const DecodeSmem& s, const uint8_t* tile,
                                             uint4 desc, int lane_koff, const TabBase& tb,
                                             int lane, float (&C)[2][4]) {
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int r = 0; r < 4; ++r) C[mt][r] = 0.f;
  const int nk16 = (desc.x >> 8) & 0xff, half = (desc.x >> 16) & 1;
  const bool split = (desc.x >> 4) & 1;
  const uint4* qf = &s.qf[desc.z][lane];
  int off = (int)desc.y + lane_koff;
#pragma unroll 1
  for (int k = 0; k < nk16; ++k, off += 128 * W, qf += 32) {
    uint32_t xa[2], xb[2];
    load_slot<W>(tile, off, xa);
    load_slot<W>(tile, off + 64 * W, xb);
    const uint4 qv = *qf;
#define GTQ_KMT(MT)                                                  \
  {                                                                  \
    uint32_t ah[4], al[4];                                           \
    code_pair<W, 2 * (MT), true>(xa, tb, ah[0], al[0]);              \
    code_pair<W, 2 * (MT) + 1, true>(xa, tb, ah[1], al[1]);          \
    code_pair<W, 2 * (MT), true>(xb, tb, ah[2], al[2]);              \
    code_pair<W, 2 * (MT) + 1, true>(xb, tb, ah[3], al[3]);          \
    mma16816(C[MT], ah, qv.x, qv.y);                                 \
    if (split) {                                                     \
      mma16816(C[MT], ah, qv.z, qv.w);                               \
      mma16816(C[MT], al, qv.x, qv.y);                               \
    }                                                                \
  }
    GTQ_KMT(0) GTQ_KMT(1)
#undef GTQ_KMT
  }
  if (half) {
    uint32_t xa[2];
    load_slot<W>(tile, off, xa);
    const uint4 qv = *qf;
    uint32_t h0, l0, h1, l1, h2, l2, h3, l3;
    code_pair<W, 0, true>(xa, tb, h0, l0);
    code_pair<W, 1, true>(xa, tb, h1, l1);
    code_pair<W, 2, true>(xa, tb, h2, l2);
    code_pair<W, 3, true>(xa, tb, h3, l3);
    mma1688(C[0], h0, h1, qv.x);
    mma1688(C[1], h2, h3, qv.x);
    if (split) {
      mma1688(C[0], h0, h1, qv.z);
      mma1688(C[1], h2, h3, qv.z);
      mma1688(C[0], l0, l1, qv.x);
      mma1688(C[1], l2, l3, qv.x);
    }
  }
}

// P.V for one dim tile and this warp's 32 tokens: 16 codes of width VB per lane
// (pairs 8 wh .. 8 wh + 7 of the lane's 32-code portion), 2 token k-tiles
template <int VB>
__device__ __forceinline__ void value_tile(const uint8_t* lane_codes, int wh, const TabBase& tb,
                                           const uint32_t (&PB)[2][2], float (&o)[4]) {
  constexpr int NW = (16 * VB + 31) / 32 + 1;
  uint32_t x[NW];
  {
    const int byte_off = 2 * VB * wh;
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(lane_codes + (byte_off & ~3));
    const uint32_t sh = (uint32_t)(byte_off & 3) << 3;
#pragma unroll
    for (int i = 0; i < NW; ++i) x[i] = wp[i];
#pragma unroll
    for (int i = 0; i + 1 < NW; ++i) x[i] = __funnelshift_r(x[i], x[i + 1], sh);
  }
  uint32_t dummy;
#define GTQ_V_KTILE(KK)                                      \
  {                                                          \
    uint32_t av[4];                                          \
    code_pair<VB, 4 * (KK), false>(x, tb, av[0], dummy);     \
    code_pair<VB, 4 * (KK) + 1, false>(x, tb, av[1], dummy); \
    code_pair<VB, 4 * (KK) + 2, false>(x, tb, av[2], dummy); \
    code_pair<VB, 4 * (KK) + 3, false>(x, tb, av[3], dummy); \
    mma16816(o, av, PB[KK][0], PB[KK][1]);                   \
  }
  GTQ_V_KTILE(0) GTQ_V_KTILE(1)
#undef GTQ_V_KTILE
}

// Arrival of this CTA at a merge ticket after its partial is stored: true in
// every thread of the CTA that arrived last (of `count`); that CTA also resets
// the ticket for the next call.  The atomic is acquire-release at GPU scope:
// it publishes this CTA's stores (ordered before it by the CTA barrier) and,
// in the last arriver, makes the others' stores visible to its loads.
__device__ bool arrive_last(unsigned* ticket, unsigned count, int* flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned prev;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(prev) : "l"(ticket) : "memory");
    const int last = prev == count - 1;
    if (last) asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(ticket) : "memory");
    *flag = last;
  }
  __syncthreads();
  return *reinterpret_cast<volatile int*>(flag) != 0;
}

// Merge partials [first, first + count) (count <= kMergeGroup) of the 8 query
// heads: M = max m_j, L = sum 2^(m_j - M) l_j, o = sum 2^(m_j - M) o_j.  Written
// as a partial to dst (global) or, normalised (o / L), to o_rot (shared) with
// (M, L) to hm / hl.  Warp w0 + i takes query head i (and i + warps), lane = 4 dims: whole
// partial rows (coalesced), every load in flight at once, one pass.  Partials
// come from other CTAs: loads bypass L1.  The caller synchronises afterwards.
__device__ __noinline__ void merge_partials(const float* head_parts, int first, int count,
                                            float* dst, float (*o_rot)[kD], float* hm, float* hl,
                                            int w0 = 0) {
  const int lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  // warp w0 takes head 0: two merges with different w0 run side by side
  for (int hh = ((threadIdx.x >> 5) - w0 % nwarps + nwarps) % nwarps; hh < 8; hh += nwarps) {
    float2 ml[kMergeGroup];
    float4 oj[kMergeGroup];
#pragma unroll
    for (int j = 0; j < kMergeGroup; ++j) {
      ml[j] = make_float2(-1e30f, 0.f);
      oj[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < count) {
        const float* pj = head_parts + ((size_t)(first + j) * 8 + hh) * kPartialStride;
        ml[j] = __ldcg(reinterpret_cast<const float2*>(pj));
        oj[j] = __ldcg(reinterpret_cast<const float4*>(pj + 4) + lane);
      }
    }
    float M = ml[0].x;
#pragma unroll
    for (int j = 1; j < kMergeGroup; ++j) M = fmaxf(M, ml[j].x);
    float L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMergeGroup; ++j) {
      const float w = exp2f(ml[j].x - M);
      L = fmaf(w, ml[j].y, L);
      o.x = fmaf(w, oj[j].x, o.x);
      o.y = fmaf(w, oj[j].y, o.y);
      o.z = fmaf(w, oj[j].z, o.z);
      o.w = fmaf(w, oj[j].w, o.w);
    }
    if (dst) {
      float* pd = dst + hh * kPartialStride;
      reinterpret_cast<float4*>(pd + 4)[lane] = o;
      if (lane == 0) *reinterpret_cast<float2*>(pd) = make_float2(M, L);
    } else {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      *reinterpret_cast<float4*>(&o_rot[hh][4 * lane]) =
          make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      if (lane == 0) {  // (M, L) of the whole cache, for the window's combination
        hm[hh] = M;
        hl[hh] = L;
      }
    }
  }
}

// Where tile t of a head lives: contiguous per head, or (paged) page
// pages[t] of the pool, which holds one tile of every KV head of the sequence.
struct HeadView {
  const uint8_t* base;    // contiguous layout: the head's first tile
  const int32_t* pages;   // paged layout: the sequence's row of the block table
  int64_t page_stride;    // bytes per page
  int64_t head_off;       // bytes of this head within a page
  int tile_bytes;
  __device__ __forceinline__ const uint8_t* tile(const uint8_t* packed, int64_t t) const {
    if (pages) return packed + (int64_t)pages[t] * page_stride + head_off;
    return base + t * (int64_t)tile_bytes;
  }
};

// Window rows are attended in blocks of 32 by up to kWinWarps warps of each of
// the first n_w splits; a block's K and V rows are staged in shared memory with
// a padded row (conflict-free ldmatrix), then processed like a tile half of
// the cache: scores by mma (K fp16 exact, q as fp16 hi + lo), online softmax
// in base 2, P.V with A = V^T from a transposing ldmatrix, all in the original
// basis.
constexpr int kWinRowBytes = 2 * kD + 16;
constexpr int kWinBufBytes = 2 * 32 * kWinRowBytes;  // K and V rows of one block
constexpr int kWinWarps = 3;
constexpr int kWinBytes = kWinWarps * kWinBufBytes + kWinWarps * 8 * kWoStride * 4;
static_assert(kWinBytes <= kPackArea, "window staging fits in the rotation pack's area");
static_assert(kWindowPartials <= kMergeGroup, "window partials merge in one pass");

struct WindowArgs {
  const __half* rk;
  const __half* rv;
  int64_t rs0, rs1, rs2;
};

// Window rows of sequence b (clamped to [0, rlen]).
__device__ __forceinline__ int64_t window_len(const int32_t* rlens, int rlen, int b) {
  if (rlen <= 0) return 0;
  return rlens ? min(max((int64_t)rlens[b], (int64_t)0), (int64_t)rlen) : (int64_t)rlen;
}

// The window's B fragments of q in the original basis, times log2(e) / sqrt(d),
// as fp16 hi and lo, from the raw queries in qb (consumer threads).
__device__ __noinline__ void window_fragments(DecodeSmem& s, int q_fp32, int gq, int nct) {
  const float qs = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
  for (int idx = threadIdx.x; idx < 8 * 32; idx += nct) {
    const int kt = idx >> 5, ln = idx & 31, gg = ln >> 2, tt = ln & 3;
    uint32_t o4[4];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int d = (gg << 7) | (16 * kt + 2 * tt + 8 * hf);
      float v0 = 0.f, v1 = 0.f;
      if (gg < gq) {
        if (q_fp32) {
          v0 = (&s.qb[0][0])[d];
          v1 = (&s.qb[0][0])[d + 1];
        } else {
          v0 = __half2float(reinterpret_cast<const __half*>(&s.qb[0][0])[d]);
          v1 = __half2float(reinterpret_cast<const __half*>(&s.qb[0][0])[d + 1]);
        }
      }
      v0 *= qs;
      v1 *= qs;
      const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
      o4[hf] = pack_half2(h0, h1);
      o4[2 + hf] = pack_half2(__float2half_rn(v0 - __half2float(h0)), __float2half_rn(v1 - __half2float(h1)));
    }
    s.wqf[kt][ln] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
  }
}

// This split's window blocks j = split + k n_w (32 rows each) -> partial
// (m, l, o) of the 8 query heads at dst, in the layout of a split's partial.
// Every consumer thread calls it during setup, after the query rotation: it
// stages rows in `area` (the rotation pack's area, free by then and not yet
// handed to the producer), reads the window's q fragments (wqf) and uses the
// warp tables.
__device__ __noinline__ void window_pass(const WindowArgs a, DecodeSmem& s, int b, int h,
                                         int split, int n_w, int64_t wl, int ncw, uint8_t* area,
                                         uint32_t area_sa, float* dst) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int nct = ncw * 32, nww = min(ncw, kWinWarps);
  float* wo2 = reinterpret_cast<float*>(area + kWinWarps * kWinBufBytes);  // [warp][head][kWoStride]
  if (warp < nww) {
    uint8_t* kbuf = area + warp * kWinBufBytes;
    uint8_t* vbuf = kbuf + 32 * kWinRowBytes;
    const uint32_t ksa = area_sa + (uint32_t)(warp * kWinBufBytes), vsa = ksa + 32 * kWinRowBytes;
    const __half* kr = a.rk + b * a.rs0 + h * a.rs1;
    const __half* vr = a.rv + b * a.rs0 + h * a.rs1;
    float mrun[2] = {-1e30f, -1e30f}, lrun[2] = {0.f, 0.f};
    float O[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) O[i][0] = O[i][1] = O[i][2] = O[i][3] = 0.f;
    for (int k = warp;; k += nww) {
      const int64_t r0 = 32 * ((int64_t)split + (int64_t)k * n_w);
      if (r0 >= wl) break;
      // rows r0 .. r0 + 31 (zero past the window's length)
      for (int c = lane; c < 32 * 16; c += 32) {
        const int row = c >> 4, col = c & 15;
        uint4 kq = make_uint4(0u, 0u, 0u, 0u), vq = kq;
        if (r0 + row < wl) {
          kq = __ldg(reinterpret_cast<const uint4*>(kr + (r0 + row) * a.rs2 + 8 * col));
          vq = __ldg(reinterpret_cast<const uint4*>(vr + (r0 + row) * a.rs2 + 8 * col));
        }
        *reinterpret_cast<uint4*>(kbuf + row * kWinRowBytes + 16 * col) = kq;
        *reinterpret_cast<uint4*>(vbuf + row * kWinRowBytes + 16 * col) = vq;
      }
      __syncwarp();
      // scores: rows 16 mt + g (+ 8), heads 2t, 2t + 1; A = K rows (ldmatrix: matrix
      // lane >> 3 holds rows + 8 (bit 0) and dims + 8 (bit 1))
      float S_[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        S_[mt][0] = S_[mt][1] = S_[mt][2] = S_[mt][3] = 0.f;
        const uint32_t arow = ksa + (uint32_t)((16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1)) * kWinRowBytes);
#pragma unroll
        for (int kt = 0; kt < 8; ++kt) {
          uint32_t av[4];
          asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                       : "=r"(av[0]), "=r"(av[1]), "=r"(av[2]), "=r"(av[3])
                       : "r"(arow + (uint32_t)((2 * kt + (lane >> 4)) * 16))
                       : "memory");
          const uint4 qv = s.wqf[kt][lane];
          mma16816(S_[mt], av, qv.x, qv.y);
          mma16816(S_[mt], av, qv.z, qv.w);
        }
      }
      // online softmax over the block (rows past the window are -inf)
      const bool full = r0 + 32 <= wl;
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int j = 16 * mt + g + 8 * (r >> 1);
          if (!full && r0 + j >= wl) S_[mt][r] = -INFINITY;
          mx[r & 1] = fmaxf(mx[r & 1], S_[mt][r]);
        }
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        mx[q2] = fmaxf(mx[q2], __shfl_xor_sync(0xffffffffu, mx[q2], 4));
        mx[q2] = fmaxf(mx[q2], __shfl_xor_sync(0xffffffffu, mx[q2], 8));
        mx[q2] = fmaxf(mx[q2], __shfl_xor_sync(0xffffffffu, mx[q2], 16));
      }
      float alpha[2];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const float mn = fmaxf(mrun[q2], mx[q2]);
        alpha[q2] = exp2f(mrun[q2] - mn);
        mrun[q2] = mn;
        lrun[q2] *= alpha[q2];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        O[i][0] *= alpha[0];
        O[i][2] *= alpha[0];
        O[i][1] *= alpha[1];
        O[i][3] *= alpha[1];
      }
      uint32_t PB[2][2];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        float pp[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          pp[r] = exp2f(S_[mt][r] - mrun[r & 1]);
          lrun[r & 1] += pp[r];
        }
        PB[mt][0] = movmatrix_t(pack_half2(__float2half_rn(pp[0]), __float2half_rn(pp[1])));
        PB[mt][1] = movmatrix_t(pack_half2(__float2half_rn(pp[2]), __float2half_rn(pp[3])));
      }
      // P.V: A = V^T (16 dims x 16 rows) by a transposing ldmatrix
      const uint32_t vrow = vsa + (uint32_t)(((lane & 7) + 8 * (lane >> 4)) * kWinRowBytes);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint32_t av[4];
          ldmatrix_x4_trans(av, vrow + (uint32_t)(kk * 16 * kWinRowBytes + (2 * i + ((lane >> 3) & 1)) * 16));
          mma16816(O[i], av, PB[kk][0], PB[kk][1]);
        }
      __syncwarp();  // the block's rows are read before the next block lands
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 4);
      lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 8);
      lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 16);
    }
    if (g == 0) {
      *reinterpret_cast<float2*>(&s.wm[warp][2 * t]) = make_float2(mrun[0], mrun[1]);
      *reinterpret_cast<float2*>(&s.wl[warp][2 * t]) = make_float2(lrun[0], lrun[1]);
    }
    float* o0 = wo2 + (warp * 8 + 2 * t) * kWoStride;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o0[16 * i + g] = O[i][0];
      o0[kWoStride + 16 * i + g] = O[i][1];
      o0[16 * i + g + 8] = O[i][2];
      o0[kWoStride + 16 * i + g + 8] = O[i][3];
    }
  }
  consumers_sync(nct);
  if (tid < 8) {
    const int hh = tid;
    float M = -1e30f;
    for (int w = 0; w < nww; ++w) M = fmaxf(M, s.wm[w][hh]);
    float L = 0.f;
    for (int w = 0; w < nww; ++w) {
      const float sc = exp2f(s.wm[w][hh] - M);
      s.wsc[w][hh] = sc;
      L = fmaf(sc, s.wl[w][hh], L);
    }
    *reinterpret_cast<float2*>(dst + hh * kPartialStride) = make_float2(M, L);
  }
  consumers_sync(nct);
  for (int idx = tid; idx < 8 * kD / 4; idx += nct) {
    const int hh = idx >> 5, d4 = idx & 31;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int w = 0; w < nww; ++w) {
      const float sc = s.wsc[w][hh];
      const float4 x = *reinterpret_cast<const float4*>(wo2 + (w * 8 + hh) * kWoStride + 4 * d4);
      v.x = fmaf(sc, x.x, v.x);
      v.y = fmaf(sc, x.y, v.y);
      v.z = fmaf(sc, x.z, v.z);
      v.w = fmaf(sc, x.w, v.w);
    }
    *reinterpret_cast<float4*>(dst + hh * kPartialStride + 4 + 4 * d4) = v;
  }
  consumers_sync(nct);  // the staging area is free again
}

// WIN: a window of fp16 rows may be attended (a separate instantiation, so that
// decodes without one carry none of its code)
template <int VB, bool WIN>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap vmap, DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem& s = *reinterpret_cast<DecodeSmem*>(smem_raw);
  const uint32_t raw_sa = smem_u32(smem_raw);
  uint8_t* tab = smem_raw + (kTabSharedAddr - raw_sa);
  // value rows (K-only plans) land with the 128-byte swizzle: 1024-byte stages
  constexpr uint32_t kStageAlign = VB > 0 ? 128u : 1024u;
  const uint32_t stage_sa =
      (raw_sa + (uint32_t)sizeof(DecodeSmem) + kStageAlign - 1) & ~(kStageAlign - 1);
  uint8_t* stages = smem_raw + (stage_sa - raw_sa);
  const int area = (int)(kTabSharedAddr - stage_sa);  // bytes of the stage area
  float* pack = reinterpret_cast<float*>(stages + area - kPackArea);  // rotation pack at setup
  // unit = (KV head, slice of at most kQSlice of its query heads); every unit
  // streams its KV head's cache and keeps its own partials and tickets
  const int unit = blockIdx.x, split = blockIdx.y, nsplit = gridDim.y;
  const int head = unit / a.nqs, qs = unit - head * a.nqs;
  const int gq = min(kQSlice, a.gq - kQSlice * qs);  // query heads of this slice
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int np = a.np, ncw = 2 * np, S = a.ring;
  const bool producer = warp == ncw;
  const int b = head / a.hkv, h = head % a.hkv;
  // the host planned the stage ring for a window that starts at or below
  // shared address 1024; anything else is reported and nothing is touched
  if (raw_sa > 1024u || area < S * a.stride || area < kTailBytes) {
    if (tid == 0) atomicOr(a.status, kStatusLayout);
    return;
  }

  HeadView hv;
  hv.tile_bytes = a.tile_bytes;
  hv.pages = a.block_table ? a.block_table + (int64_t)b * a.max_blocks : nullptr;
  hv.page_stride = (int64_t)a.hkv * a.tile_bytes;
  hv.head_off = (int64_t)h * a.tile_bytes;
  hv.base = a.packed + (size_t)head * a.n_tiles * a.tile_bytes;

  if (tid == 0) {
    mbar_init(&s.tab_bar, 1);
    mbar_init(&s.meta_bar, 1);
    mbar_init(&s.pack_bar, 1);
    mbar_init(&s.done_bar, 1);
    mbar_init(&s.rv_bar, 1);
    for (int i = 0; i < S; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 2 * kTPS);
    }
    s.failed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // the tables are the library's constants: safe to read before the wait
    mbar_expect_tx(&s.tab_bar, (unsigned)kDecodeImageBytes);
    bulk_copy(tab, a.dec_image, kDecodeImageBytes, &s.tab_bar);
  }
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();  // queries, metadata and the cache may come from the previous grid
  if (tid == 0) {
    // the metadata, the first part of the rotation pack and the unit's gq
    // queries (contiguous) land on one barrier; the queries go to qb as they are
    const unsigned esz = a.q_fp32 ? 4u : 2u, qbytes = (unsigned)gq * kD * esz;
    mbar_expect_tx(&s.meta_bar, (unsigned)(sizeof(HeadMeta) + kPackPrefix) + qbytes);
    bulk_copy(&s.meta, a.meta + head, sizeof(HeadMeta), &s.meta_bar);
    bulk_copy(pack, a.rotpack + (size_t)head * kRotPackMaxWords, kPackPrefix, &s.meta_bar);
    bulk_copy(&s.qb[0][0],
              reinterpret_cast<const uint8_t*>(a.q) +
                  (((size_t)b * a.hkv + h) * a.gq + (size_t)kQSlice * qs) * kD * esz,
              qbytes,
              &s.meta_bar);
  }
  const int64_t T = a.seq_lens ? min((int64_t)a.seq_lens[b], a.T) : a.T;
  const int64_t tiles_T = (max(T, (int64_t)0) + kTile - 1) / kTile;
  unsigned* head_tickets = a.tickets + (size_t)unit * kTicketStride;
  bool failed = false;

  // per-warp running state (consumers; set just before the tile loop)
  float mrun[2] = {-1e30f, -1e30f}, lrun[2] = {0.f, 0.f};
  float O[8][4];

  // the window rows this split will attend: into L2 now
  const int64_t wl = WIN ? window_len(a.rlens, a.rlen, b) : 0;
  const int n_w = WIN ? (int)min((int64_t)min(nsplit, kWindowPartials), (wl + 31) / 32) : 0;
  if (producer && lane == 0 && split < n_w && a.rs2 == kD)
    for (int64_t r0 = 32 * (int64_t)split; r0 < wl; r0 += 32 * (int64_t)n_w) {
      const unsigned bytes = (unsigned)(min((int64_t)32, wl - r0) * kD * 2);
      prefetch_l2(a.rk + b * a.rs0 + h * a.rs1 + r0 * kD, bytes);
      prefetch_l2(a.rv + b * a.rs0 + h * a.rs1 + r0 * kD, bytes);
    }
  if (producer) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the schedule (lane 0's counter grabs are broadcast);
    // lane 0 issues the stage copies.
    {
      int fills = 0;
      if (!__all_sync(0xffffffffu, mbar_wait(&s.meta_bar, 0))) {
        failed = true;
      } else {
        const int load_bytes = key_norm_offset(a.kb, VB) + 128 * s.meta.n_groups;
        const int pack_lo = area - kPackArea;
        const uint64_t pol = evict_first_policy();
        unsigned* ctr = head_tickets + kSchedWord;
        // static share first; the counter's grabs are issued ahead of use, so
        // their round trip never holds up a load
        const int64_t st0 = min((int64_t)split * a.static_per, tiles_T);
        const int64_t st1 = min(st0 + a.static_per, tiles_T);
        const int64_t dyn0 = (int64_t)nsplit * a.static_per;
        int64_t snext = st0;
        bool setup_ok = false, exhausted = false;
        auto grab = [&]() -> int {
          int v = 0;
          if (lane == 0) v = (int)atomicAdd(ctr, (unsigned)kGrab);
          return __shfl_sync(0xffffffffu, v, 0);
        };
        int g0 = grab(), g1 = grab();
        int used = 0;
        auto next_tile = [&]() -> int64_t {
          if (snext < st1) return snext++;
          if (exhausted) return -1;
          if (used == kGrab) {
            g0 = g1;
            used = 0;
            if (dyn0 + g0 < tiles_T) g1 = grab();
          }
          const int64_t t = dyn0 + g0 + used++;
          if (t >= tiles_T) {
            exhausted = true;
            return -1;
          }
          return t;
        };
        int64_t pending = next_tile();
        int ends = 0, slot = 0, round = 0;
        for (;; ++fills) {
          if (round > 0 &&
              !__all_sync(0xffffffffu, mbar_wait(&s.empty[slot], (unsigned)(round - 1) & 1u))) {
            failed = true;
            break;
          }
          if (!setup_ok && (slot + 1) * a.stride > pack_lo) {
            if (!__all_sync(0xffffffffu, mbar_wait(&s.done_bar, 0))) {
              failed = true;
              break;
            }
            setup_ok = true;
          }
          uint8_t* dst = stages + (size_t)slot * a.stride;
          if (pending >= 0) {
            const int64_t t0 = pending;
            pending = next_tile();
            int64_t t1 = kSkip;
            if (pending == t0 + 1) {
              t1 = pending;
              pending = next_tile();
            }
            if (lane == 0) {
              s.stage_tile[slot] = make_int2((int)t0, (int)t1);
              // K-only: 16 KB of fp16 value rows per tile (zero past the call's T)
              const unsigned vbytes = VB > 0 ? 0u : (t1 >= 0 ? 2u : 1u) * (unsigned)(kTile * kD * 2);
              if (t1 >= 0 && !hv.pages) {  // adjacent tiles: one copy
                mbar_expect_tx(&s.full[slot], (unsigned)(a.tile_bytes + load_bytes) + vbytes);
                bulk_copy_hint(dst, hv.tile(a.packed, t0), (unsigned)(a.tile_bytes + load_bytes),
                               &s.full[slot], pol);
              } else {
                mbar_expect_tx(&s.full[slot],
                               (unsigned)(t1 >= 0 ? 2 * load_bytes : load_bytes) + vbytes);
                bulk_copy_hint(dst, hv.tile(a.packed, t0), (unsigned)load_bytes, &s.full[slot], pol);
                if (t1 >= 0)
                  bulk_copy_hint(dst + a.tile_bytes, hv.tile(a.packed, t1), (unsigned)load_bytes,
                                 &s.full[slot], pol);
              }
              if (VB == 0) {
                // rows of tile tt: box (64 dims, 64 tokens, both dim halves) -> [half][token][64]
                auto load_values = [&](uint8_t* vdst, int64_t tt) {
                  const int row = (int)(tt * kTile);
                  if (a.v_loads == 1) {
                    tma_load_5d(vdst, &vmap, 0, row, 0, h, b, &s.full[slot]);
                  } else {
                    tma_load_4d(vdst, &vmap, 0, row, h, b, &s.full[slot]);
                    tma_load_4d(vdst + kTile * 128, &vmap, 64, row, h, b, &s.full[slot]);
                  }
                };
                load_values(dst + a.voff, t0);
                if (t1 >= 0) load_values(dst + a.voff + kTile * kD * 2, t1);
              }
            }
          } else {
            // end markers: every pair meets one as its next tile slot
            if (lane == 0) {
              s.stage_tile[slot] = make_int2(kEnd, kEnd);
              mbar_arrive(&s.full[slot]);
            }
            ends += kTPS;
            if (ends >= np) {
              ++fills;
              break;
            }
          }
          if (++slot == S) {
            slot = 0;
            ++round;
          }
        }
        asm volatile("" ::"r"(g0), "r"(g1));  // every grab has returned before the CTA moves on
      }
      // drain: no bulk copy into this CTA's shared memory may outlive the loop
      if (lane == 0) {
        const int n_used = min(fills, S);
        for (int sl = 0; sl < n_used; ++sl) {
          const int last = sl + ((fills - 1 - sl) / S) * S;  // last fill index of the slot
          mbar_wait(&s.full[sl], (unsigned)(last / S) & 1u);
        }
      }
      if (failed && lane == 0) s.failed = 1;
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int nct = ncw * 32;
    const int g = lane >> 2, t = lane & 3;
    const int pair = warp >> 1, wh = warp & 1;
    failed = !mbar_wait(&s.meta_bar, 0);
    const HeadMeta& m = s.meta;
    if (tid == 0) {
      int words = kRotPackHeaderWords;
      for (int gi = 0; gi < m.n_groups; ++gi) words += (int)m.grp_m[gi] * m.grp_m[gi];
      const int bytes = (words * 4 + 15) & ~15;
      if (!failed && bytes > kPackPrefix) {
        mbar_expect_tx(&s.pack_bar, (unsigned)(bytes - kPackPrefix));
        bulk_copy(reinterpret_cast<uint8_t*>(pack) + kPackPrefix,
                  reinterpret_cast<const uint8_t*>(a.rotpack + (size_t)head * kRotPackMaxWords) +
                      kPackPrefix,
                  (unsigned)(bytes - kPackPrefix), &s.pack_bar);
      } else {
        mbar_arrive(&s.pack_bar);
      }
    }
    failed = !mbar_wait(&s.pack_bar, 0) || failed;
    // gather, transposed: qT[p][hh] = q[hh][dim of group coordinate p] (zero past
    // the group size and the slots); qT lives in qa, the raw queries in qb
    float(*qT)[8] = reinterpret_cast<float(*)[8]>(&s.qa[0][0]);
    const uint8_t* coord_dim = reinterpret_cast<const uint8_t*>(pack);
    for (int i = tid; i < 8 * kD; i += nct) {
      const int p = i >> 3, hh = i & 7;
      float v = 0.f;
      if (hh < gq && (p >> 1) < m.n_slots) {
        const int d = (hh << 7) | (coord_dim[p] & (kD - 1));
        v = a.q_fp32 ? (&s.qb[0][0])[d] : __half2float(reinterpret_cast<const __half*>(&s.qb[0][0])[d]);
      }
      qT[p][hh] = v;
    }
    if (split < n_w) window_fragments(s, a.q_fp32, gq, nct);  // before the rotation overwrites qb
    consumers_sync(nct);
    // q_rot[hh][pos] = sum_c R_g[r][c] qT[first + c][hh] * log2(e) / (sqrt(d) sqrt(m_g)),
    // into qb: a task is one position and four heads
    for (int task = tid; task < 2 * kD; task += nct) {
      const int pos = task & (kD - 1), h4 = (task >> 7) * 4, slot = pos >> 1;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      float sc = 0.f;
      if (slot < m.n_slots) {
        const int gi = m.slot_group[slot], mm = m.grp_m[gi];
        const int first = 2 * m.grp_first_slot[gi], r = pos - first;
        int off = kRotPackHeaderWords;
        for (int gg = 0; gg < gi; ++gg) off += (int)m.grp_m[gg] * m.grp_m[gg];
        const float* Rc = pack + off + r;
        const float4* qc = reinterpret_cast<const float4*>(&qT[first][h4]);
#pragma unroll 4
        for (int c = 0; c < mm; ++c) {
          const float rv = Rc[c * mm];
          const float4 qv = qc[2 * c];
          acc.x = fmaf(rv, qv.x, acc.x);
          acc.y = fmaf(rv, qv.y, acc.y);
          acc.z = fmaf(rv, qv.z, acc.z);
          acc.w = fmaf(rv, qv.w, acc.w);
        }
        sc = m.inv_sqrt_m[gi] * (1.4426950408889634f * 0.08838834764831845f);
      }
      s.qb[h4][pos] = acc.x * sc;
      s.qb[h4 + 1][pos] = acc.y * sc;
      s.qb[h4 + 2][pos] = acc.z * sc;
      s.qb[h4 + 3][pos] = acc.w * sc;
    }
    consumers_sync(nct);
    // the first n_w splits attend the fp16 window's 32-row blocks now, staged in
    // the pack's area, each into a window partial of its own
    if (split < n_w) {
      const WindowArgs wa = {a.rk, a.rv, a.rs0, a.rs1, a.rs2};
      window_pass(wa, s, b, h, split, n_w, wl, ncw, reinterpret_cast<uint8_t*>(pack), smem_u32(pack),
                  a.partials + ((size_t)unit * a.slot_total + a.slot_window + split) * 8 * kPartialStride);
    }
    if (tid == 0) mbar_arrive(&s.done_bar);  // the pack's stages may be filled now
    // group descriptors: W | split << 4 | k16 tiles << 8 | half k-tile << 16
    if (tid < m.n_groups) {
      const int gi = tid, cnt = m.grp_m[gi] >> 1, rem = cnt & 7;
      const int k16 = cnt / 8 + (rem > 4 ? 1 : 0), half = (rem >= 1 && rem <= 4) ? 1 : 0;
      s.gdesc[gi] = make_uint4((uint32_t)m.grp_width[gi] | ((uint32_t)(m.grp_split[gi] & 1) << 4) |
                                   ((uint32_t)k16 << 8) | ((uint32_t)half << 16),
                               (uint32_t)m.slot_koff[m.grp_first_slot[gi]], (uint32_t)m.grp_kt0[gi],
                               0u);
    }
    // B fragments (query) of every decode k-tile; slots past the k-tile's run are zero
    for (int idx = tid; idx < m.n_ktiles * 32; idx += nct) {
      const int kt = idx >> 5, ln = idx & 31, gg = ln >> 2, tt = ln & 3;
      uint32_t outv[4];
      for (int hf = 0; hf < 2; ++hf) {
        const int sl = tt + 4 * hf;  // slot within the k-tile
        const bool in = sl < m.kt_nslots[kt];
        const int pos = 2 * (m.kt_first_slot[kt] + sl);
        const float v0 = in ? s.qb[gg][pos] : 0.f, v1 = in ? s.qb[gg][pos + 1] : 0.f;
        const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
        outv[hf] = pack_half2(h0, h1);
        outv[2 + hf] = pack_half2(__float2half_rn(v0 - __half2float(h0)),
                                  __float2half_rn(v1 - __half2float(h1)));
      }
      s.qf[kt][ln] = make_uint4(outv[0], outv[1], outv[2], outv[3]);
    }
    failed = !mbar_wait(&s.tab_bar, 0) || failed;
    consumers_sync(nct);

    const int n_groups = m.n_groups;
    const int kb = a.kb;
    const int load_v = 1024 * kb;
    const int vnorm_off = value_norm_offset(kb, VB), knorm_off = key_norm_offset(kb, VB);
    TabBase tb;
    tb.bss = kTabSharedAddr;
    tb.b32 = kTabSharedAddr | ((uint32_t)lane << 2);
    tb.b16 = kTabSharedAddr | ((uint32_t)(lane & 15) << 3);
    // lane portion of slot t: 16W bits at byte 16W t + 2W g; this warp's half: + W wh
    const int lane_kunit = 16 * t + 2 * g + wh;  // times W

#pragma unroll
    for (int i = 0; i < 8; ++i) O[i][0] = O[i][1] = O[i][2] = O[i][3] = 0.f;
    // tile slot j = pair + k np of the stage sequence: stage j / kTPS, slot j % kTPS
    int j = pair, fi = pair / kTPS, slot = fi % S, round = fi / S;
    // a timeout seen by any lane stops the whole warp (the loop body is warp-wide)
    failed = __any_sync(0xffffffffu, failed);
    while (!failed) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s.full[slot], (unsigned)round & 1u))) {
        failed = true;
        break;
      }
      const int2 st2 = s.stage_tile[slot];
      const int jk = j % kTPS;
      const int tile_idx = jk ? st2.y : st2.x;
      if (tile_idx == kEnd) break;
      auto advance = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty[slot]);
        j += np;
        const int nfi = j / kTPS;
        slot += nfi - fi;
        fi = nfi;
        while (slot >= S) {
          slot -= S;
          ++round;
        }
      };
      if (tile_idx == kSkip) {
        advance();
        continue;
      }
      const uint8_t* tl = stages + (size_t)slot * a.stride + (size_t)jk * a.tile_bytes;

      // ------------------------------------------------------------ scores
      float S_[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 4; ++r) S_[mt][r] = 0.f;
#pragma unroll 1
      for (int gi = 0; gi < n_groups; ++gi) {
        const uint4 desc = s.gdesc[gi];
        float C[2][4];
        switch (desc.x & 0xf) {  // W
#define GTQ_GROUP(WW)                                                   \
  case WW:                                                              \
    group_scores<WW>(s, tl, desc, WW * lane_kunit, tb, lane, C);        \
    break;
          GTQ_GROUP(1) GTQ_GROUP(2) GTQ_GROUP(3) GTQ_GROUP(4)
          GTQ_GROUP(5) GTQ_GROUP(6) GTQ_GROUP(7) GTQ_GROUP(8)
#undef GTQ_GROUP
          default:
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
              for (int r = 0; r < 4; ++r) C[mt][r] = 0.f;
            break;
        }
        // group complete: scale by its fp16 norms (tokens g + 8u, u = 4wh .. 4wh + 3)
        const uint2 nq = *reinterpret_cast<const uint2*>(tl + knorm_off + gi * 128 + g * 16 + wh * 8);
        const __half2* nh = reinterpret_cast<const __half2*>(&nq);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const float2 n = __half22float2(nh[mt]);
          S_[mt][0] = fmaf(n.x, C[mt][0], S_[mt][0]);
          S_[mt][1] = fmaf(n.x, C[mt][1], S_[mt][1]);
          S_[mt][2] = fmaf(n.y, C[mt][2], S_[mt][2]);
          S_[mt][3] = fmaf(n.y, C[mt][3], S_[mt][3]);
        }
      }
      // ------------------------------------------------------ online softmax
      const int64_t tok0 = (int64_t)tile_idx * kTile + 32 * wh;
      const bool full = tok0 + 32 <= T;
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int j = 16 * mt + g + 8 * (r >> 1);
          if (!full && tok0 + j >= T) S_[mt][r] = -INFINITY;
          mx[r & 1] = fmaxf(mx[r & 1], S_[mt][r]);
        }
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        mx[q2] = fmaxf(mx[q2], __shfl_xor_sync(0xffffffffu, mx[q2], 4));
        mx[q2] = fmaxf(mx[q2], __shfl_xor_sync(0xffffffffu, mx[q2], 8));
        mx[q2] = fmaxf(mx[q2], __shfl_xor_sync(0xffffffffu, mx[q2], 16));
      }
      float alpha[2];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const float mn = fmaxf(mrun[q2], mx[q2]);
        alpha[q2] = exp2f(mrun[q2] - mn);
        mrun[q2] = mn;
        lrun[q2] *= alpha[q2];
      }
      if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          O[i][0] *= alpha[0];
          O[i][2] *= alpha[0];
          O[i][1] *= alpha[1];
          O[i][3] *= alpha[1];
        }
      }
      // coded values: p times the token's fp16 norm / sqrt(d); fp16 values: p
      float2 vsc[2] = {make_float2(1.f, 1.f), make_float2(1.f, 1.f)};
      if (VB > 0) {
        const uint2 vq = *reinterpret_cast<const uint2*>(tl + vnorm_off + g * 16 + wh * 8);
        const __half2* vnh = reinterpret_cast<const __half2*>(&vq);
        const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          vsc[mt] = __half22float2(vnh[mt]);
          vsc[mt].x *= inv_sqrt_d;
          vsc[mt].y *= inv_sqrt_d;
        }
      }
      uint32_t PB[2][2];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const float2 vn = vsc[mt];
        float pp[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int j = 16 * mt + g + 8 * (r >> 1);
          const float p = exp2f(S_[mt][r] - mrun[r & 1]);
          lrun[r & 1] += p;
          const float nv = (r >> 1) ? vn.y : vn.x;
          pp[r] = (full || tok0 + j < T) ? p * nv : 0.f;
        }
        PB[mt][0] = movmatrix_t(pack_half2(__float2half_rn(pp[0]), __float2half_rn(pp[1])));
        PB[mt][1] = movmatrix_t(pack_half2(__float2half_rn(pp[2]), __float2half_rn(pp[3])));
      }
      // ---------------------------------------------------------------- P.V
      if constexpr (VB > 0) {
        const uint8_t* vcodes = tl + load_v;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          value_tile<VB>(vcodes + ((i * 8 + g) * 4 + t) * VB * 4, wh, tb, PB, O[i]);
      } else {
        // A = V^T (16 dims x 16 tokens) by a transposing ldmatrix.x4: matrix
        // lane >> 3 holds dims + 8 (bit 0) and tokens + 8 (bit 1); the lane
        // gives the address of one token row, whose 16-byte chunks sit
        // XOR-swizzled by the row's index mod 8
        const uint32_t vrow = stage_sa + (uint32_t)(slot * a.stride + a.voff + jk * kTile * kD * 2) +
                              (uint32_t)(32 * wh + (lane & 7) + 8 * (lane >> 4)) * 128u;
        const uint32_t lx = (uint32_t)(((lane >> 3) & 1) ^ (lane & 7));
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          uint32_t m0 = 0xffffffffu, m1 = 0xffffffffu;  // rows past the sequence are zero
          if (!full) {
            const int64_t tk = tok0 + 16 * kk + 2 * t;
            m0 = (tk < T ? 0xffffu : 0u) | (tk + 1 < T ? 0xffff0000u : 0u);
            m1 = (tk + 8 < T ? 0xffffu : 0u) | (tk + 9 < T ? 0xffff0000u : 0u);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            uint32_t av[4];
            ldmatrix_x4_trans(av, vrow + (uint32_t)(kk * 16 * 128 + (i >> 2) * kTile * 128) +
                                      ((((uint32_t)(2 * i) & 7u) ^ lx) << 4));
            av[0] &= m0;
            av[1] &= m0;
            av[2] &= m1;
            av[3] &= m1;
            mma16816(O[i], av, PB[kk][0], PB[kk][1]);
          }
        }
      }
      // ---------------------------------------------------- release the stage
      advance();
    }
    if (failed && lane == 0) s.failed = 1;
    // lanes' partial l over their tokens
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 4);
      lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 8);
      lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 16);
    }
  }
  // every warp is done with the stages and the producer has drained its copies
  __syncthreads();
  if (tid == 0) {
    // the setup copies have landed (or waited out) before the area is reused
    mbar_wait(&s.meta_bar, 0);
    mbar_wait(&s.pack_bar, 0);
    mbar_wait(&s.tab_bar, 0);
  }
  __syncthreads();
  const bool cta_failed = *reinterpret_cast<volatile int*>(&s.failed) != 0;
  if (cta_failed && tid == 0) atomicOr(a.status, kStatusTimeout);

  // ------------------------------------------------- merge the warps in the CTA
  // wo[warp][head][kWoStride]: each warp's o rescaled to the CTA's maximum (the
  // padded head stride keeps a warp's fragment stores free of bank conflicts)
  float* wo = reinterpret_cast<float*>(stages);
  uint4* rvf = reinterpret_cast<uint4*>(stages + kRvOff);  // R_V^T as A fragments
  if (!producer && (lane >> 2) == 0) {
    const int t = lane & 3;
    *reinterpret_cast<float2*>(&s.wm[warp][2 * t]) = make_float2(mrun[0], mrun[1]);
    *reinterpret_cast<float2*>(&s.wl[warp][2 * t]) = make_float2(lrun[0], lrun[1]);
  }
  __syncthreads();
  if (!producer) {
    const int g = lane >> 2, t = lane & 3;
    float M0 = -1e30f, M1 = -1e30f;
    for (int w = 0; w < ncw; ++w) {
      const float2 mw = *reinterpret_cast<const float2*>(&s.wm[w][2 * t]);
      M0 = fmaxf(M0, mw.x);
      M1 = fmaxf(M1, mw.y);
    }
    const float sc0 = exp2f(mrun[0] - M0), sc1 = exp2f(mrun[1] - M1);
    float* o0 = wo + (warp * 8 + 2 * t) * kWoStride;  // head 2t; head 2t + 1 one row on
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o0[16 * i + g] = O[i][0] * sc0;
      o0[kWoStride + 16 * i + g] = O[i][1] * sc1;
      o0[16 * i + g + 8] = O[i][2] * sc0;
      o0[kWoStride + 16 * i + g + 8] = O[i][3] * sc1;
    }
    if (warp == 0 && g == 0) {  // the CTA's (M, L) of heads 2t, 2t + 1
      float L0 = 0.f, L1 = 0.f;
      for (int w = 0; w < ncw; ++w) {
        const float2 mw = *reinterpret_cast<const float2*>(&s.wm[w][2 * t]);
        const float2 lw = *reinterpret_cast<const float2*>(&s.wl[w][2 * t]);
        L0 = fmaf(exp2f(mw.x - M0), lw.x, L0);
        L1 = fmaf(exp2f(mw.y - M1), lw.y, L1);
      }
      s.hm[2 * t] = M0;
      s.hm[2 * t + 1] = M1;
      s.hl[2 * t] = L0;
      s.hl[2 * t + 1] = L1;
    }
  }
  __syncthreads();
  float* head_parts = a.partials + (size_t)unit * a.slot_total * 8 * kPartialStride;
  float* part = head_parts + (size_t)split * 8 * kPartialStride;
  // this CTA's (m, l, o_rot): the output itself with a single split, else its
  // partial in global memory; a task is 4 dims of one head
  for (int idx = tid; idx < 8 * kD / 4; idx += blockDim.x) {
    const int hh = idx >> 5, d4 = idx & 31;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kCWarps; ++w)
      if (w < ncw) {
        const float4 x = *reinterpret_cast<const float4*>(wo + (w * 8 + hh) * kWoStride + 4 * d4);
        v.x += x.x;
        v.y += x.y;
        v.z += x.z;
        v.w += x.w;
      }
    if (nsplit == 1) {
      const float inv = s.hl[hh] > 0.f ? 1.f / s.hl[hh] : 0.f;
      *reinterpret_cast<float4*>(&s.qa[hh][4 * d4]) = make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
    } else {
      *reinterpret_cast<float4*>(part + hh * kPartialStride + 4 + 4 * d4) = v;
      if (d4 == 0) *reinterpret_cast<float2*>(part + hh * kPartialStride) = make_float2(s.hm[hh], s.hl[hh]);
    }
  }
  // ---------------- merge of the splits, without waiting: the last CTA to
  // arrive in a group of kMergeGroup splits merges the group into a
  // second-level partial, and the last group to finish merges those.  A CTA
  // that may finish fetches R_V^T while it merges (coded values only).
  auto fetch_rv = [&]() -> bool {
    if (VB == 0) return false;
    if (tid == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&s.rv_bar, (unsigned)kRvFragBytes);
      bulk_copy(rvf, a.rv_frag, kRvFragBytes, &s.rv_bar);
    }
    return true;
  };
  // the window's partials merged into qb (normalised) with (M_w, L_w) in wsc[0],
  // [1], by other warps than the cache's merge (no barrier between the two)
  auto merge_window = [&]() {
    if (n_w > 0) merge_partials(head_parts, a.slot_window, n_w, nullptr, s.qb, s.wsc[0], s.wsc[1], 8);
  };
  bool finish = nsplit == 1, rv_issued = false;
  if (finish) {
    __syncthreads();
    rv_issued = fetch_rv();
    merge_window();
  } else {
    const int n_grp = (nsplit + kMergeGroup - 1) / kMergeGroup;
    const int grp = split / kMergeGroup;
    const int n1 = min(kMergeGroup, nsplit - grp * kMergeGroup);
    if (arrive_last(&head_tickets[1 + grp], (unsigned)n1, &s.flag)) {
      rv_issued = fetch_rv();
      if (n_grp == 1) {
        merge_partials(head_parts, grp * kMergeGroup, n1, nullptr, s.qa, s.hm, s.hl);
        merge_window();
        finish = true;
      } else {
        merge_partials(head_parts, grp * kMergeGroup, n1,
                       head_parts + (size_t)(a.slot_groups + grp) * 8 * kPartialStride, nullptr,
                       s.hm, s.hl);
        if (arrive_last(&head_tickets[0], (unsigned)n_grp, &s.flag)) {
          merge_partials(head_parts, a.slot_groups, n_grp, nullptr, s.qa, s.hm, s.hl);
          merge_window();
          finish = true;
        }
      }
    }
  }
  bool rv_ok = true;
  if (rv_issued) rv_ok = mbar_wait(&s.rv_bar, 0);  // no CTA exits with the copy in flight
  if (!finish) return;
  if (tid == 0)  // every CTA of the head has grabbed its last tile: reset the counter
    asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(head_tickets + kSchedWord) : "memory");
  rv_ok = __syncthreads_and(rv_ok);
  if (!rv_ok) {
    if (tid == 0) atomicOr(a.status, kStatusTimeout);
    return;
  }
  // out = cr o_cache + cw o_window (both normalised): the two softmax parts
  // weighted by their sums at their common maximum
  if (tid < 8) {
    float cr = 1.f, cw = 0.f;
    if (n_w > 0) {
      const float M = s.hm[tid], L = s.hl[tid], Mw = s.wsc[0][tid], Lw = s.wsc[1][tid];
      const float Mx = fmaxf(M, Mw);
      const float wr = exp2f(M - Mx) * L, ww = exp2f(Mw - Mx) * Lw;
      const float den = wr + ww;
      cr = den > 0.f ? wr / den : 0.f;
      cw = den > 0.f ? ww / den : 0.f;
    }
    s.wm[0][tid] = cr;
    s.wl[0][tid] = cw;
  }
  __syncthreads();
  float* out_head = a.out + (((size_t)b * a.hkv + h) * a.gq + (size_t)kQSlice * qs) * kD;
  auto window_o = [&](int hh, int dd) -> float { return n_w > 0 ? s.wl[0][hh] * s.qb[hh][dd] : 0.f; };
  if constexpr (VB == 0) {  // fp16 values: o_cache is already in the original basis
    for (int idx = tid; idx < gq * kD; idx += blockDim.x) {
      const int hh = idx >> 7, dd = idx & (kD - 1);
      out_head[idx] = fmaf(s.wm[0][hh], s.qa[hh][dd], window_o(hh, dd));
    }
  } else {
  // out[hh][dd] = sum_r R_V[r][dd] o_rot[hh][r] on the tensor cores: m-tile mt
  // (dims [16 mt, 16 mt + 16)) goes to warp mt mod warps, A = R_V^T (fp16 hi + lo fragments), B =
  // o_rot^T split into fp16 hi + lo; A_hi B_hi + A_hi B_lo + A_lo B_hi
  for (int mt = warp; mt < 8; mt += blockDim.x >> 5) {
    const int g = lane >> 2, t = lane & 3;
    // three accumulators (hi.hi, hi.lo, lo.hi), so that the mma chains overlap
    float c[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
      const uint4 fh = rvf[((mt * 8 + kt) * 32 + lane) * 2], fl = rvf[((mt * 8 + kt) * 32 + lane) * 2 + 1];
      const uint32_t ah[4] = {fh.x, fh.y, fh.z, fh.w}, al[4] = {fl.x, fl.y, fl.z, fl.w};
      const int r0 = 16 * kt + 2 * t;
      const float2 x0 = *reinterpret_cast<const float2*>(&s.qa[g][r0]);
      const float2 x1 = *reinterpret_cast<const float2*>(&s.qa[g][r0 + 8]);
      const __half h00 = __float2half_rn(x0.x), h01 = __float2half_rn(x0.y);
      const __half h10 = __float2half_rn(x1.x), h11 = __float2half_rn(x1.y);
      const uint32_t bh0 = pack_half2(h00, h01), bh1 = pack_half2(h10, h11);
      const uint32_t bl0 = pack_half2(__float2half_rn(x0.x - __half2float(h00)),
                                      __float2half_rn(x0.y - __half2float(h01)));
      const uint32_t bl1 = pack_half2(__float2half_rn(x1.x - __half2float(h10)),
                                      __float2half_rn(x1.y - __half2float(h11)));
      mma16816(c, ah, bh0, bh1);
      mma16816(c1, ah, bl0, bl1);
      mma16816(c2, al, bh0, bh1);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) c[r] += c1[r] + c2[r];
    // c[0], c[1]: dim 16 mt + g, heads 2t, 2t + 1; c[2], c[3]: dim + 8
    const int dd = 16 * mt + g;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int hh = 2 * t + (r & 1), d = dd + 8 * (r >> 1);
      if (hh < gq) out_head[hh * kD + d] = fmaf(s.wm[0][hh], c[r], window_o(hh, d));
    }
  }
  }
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace

cudaError_t launch_decode(const gtq_plan* p, const uint8_t* packed, int64_t T, const void* q,
                          int q_dtype, float* out, const SeqMap& sm, const Fp16Kv& kv,
                          cudaStream_t s) {
  DecodeArgs a;
  const bool konly = p->cfg.v_bits == 0;
  a.packed = packed;
  a.meta = p->d_meta;
  a.rotpack = p->d_rotpack;
  a.q = q;
  a.q_fp32 = q_dtype == GTQ_DTYPE_FP32;
  a.rv_frag = reinterpret_cast<const uint4*>(p->tab.rv_frag);
  a.out = out;
  a.tickets = p->d_tickets;
  a.hkv = p->cfg.n_kv_heads;
  a.gq = p->g_q;
  a.nqs = p->n_qs;
  a.dec_image = p->tab.dec_image;
  a.partials = p->d_partials;
  const int split_cap = decode_split_cap(p->n_sms, p->n_units);
  const PartialSlots slots(split_cap);
  a.slot_groups = slots.groups;
  a.slot_window = slots.window;
  a.slot_total = slots.total;
  a.status = p->d_status;
  a.seq_lens = sm.seq_lens;
  a.block_table = sm.table;
  a.max_blocks = sm.max_blocks;
  a.T = T;
  a.n_tiles = p->n_tiles;
  a.tile_bytes = (int)p->tile_bytes;
  a.kb = p->cfg.k_bits;
  // a stage: kTPS tiles, then (K-only) their fp16 value rows, 16 KB per tile
  const size_t salign = konly ? 1024 : 128;
  a.voff = (int)((kTPS * p->tile_bytes + salign - 1) & ~(salign - 1));
  a.stride = konly ? a.voff + kTPS * kTile * kD * 2 : a.voff;
  a.v_loads = 1;
  a.rk = kv.rk;
  a.rv = kv.rv;
  a.rs0 = kv.rs[0];
  a.rs1 = kv.rs[1];
  a.rs2 = kv.rs[2];
  a.rlens = kv.rlens;
  a.rlen = (int)kv.rlen;
  CUtensorMap vmap;
  memset(&vmap, 0, sizeof(vmap));
  if (konly) {
    // (64 dims, T tokens, 2 dim halves, Hkv, B): one copy per tile brings both
    // halves; without it, a 4-D map and a copy per half give the same layout
    const uint64_t dims5[5] = {64, (uint64_t)T, 2, (uint64_t)p->cfg.n_kv_heads,
                               (uint64_t)p->cfg.batch};
    const uint64_t st5[4] = {(uint64_t)kv.vs[2] * 2, 128, (uint64_t)kv.vs[1] * 2,
                             (uint64_t)kv.vs[0] * 2};
    const uint32_t box5[5] = {64, (uint32_t)kTile, 2, 1, 1};
    if (!encode_fp16_map(&vmap, 5, kv.v, dims5, st5, box5, true)) {
      const uint64_t dims4[4] = {(uint64_t)kD, (uint64_t)T, (uint64_t)p->cfg.n_kv_heads,
                                 (uint64_t)p->cfg.batch};
      const uint64_t st4[3] = {(uint64_t)kv.vs[2] * 2, (uint64_t)kv.vs[1] * 2,
                               (uint64_t)kv.vs[0] * 2};
      const uint32_t box4[4] = {64, (uint32_t)kTile, 1, 1};
      if (!encode_fp16_map(&vmap, 4, kv.v, dims4, st4, box4, true)) return cudaErrorNotSupported;
      a.v_loads = 2;
    }
  }
  int dev_smem = 0;
  cudaDeviceGetAttribute(&dev_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, p->device);
  if (dev_smem < kSmemBytes) return cudaErrorInvalidValue;
  // stage area: below the table region, after DecodeSmem (the dynamic window may
  // start up to 1 KB above shared address 0)
  const int area = (int)kTabSharedAddr - (int)((1024 + sizeof(DecodeSmem) + salign - 1) & ~(salign - 1));
  if (area < kTailBytes || area < kPackArea + a.stride) return cudaErrorInvalidValue;
  const int ring = std::min(kMaxRing, area / a.stride);
  if (ring < 2) return cudaErrorInvalidValue;
  // pairs: half the tile slots (each pair has its next tile in flight); K-only
  // stages are large (fp16 value rows), so there one pair per slot (measured
  // 22% faster at 128K; pairs take slots in order, so the producer always
  // advances)
  const int np = std::max(1, std::min(kPairs, konly ? ring * kTPS : ring * kTPS / 2));
  a.ring = ring;
  a.np = np;
  const int64_t tiles_T = (T + kTile - 1) / kTile;
  // one CTA per SM; with many heads, round up so that late CTAs join heads that
  // still have tiles left (the counter balances the work within a head)
  int splits = (int)std::min<int64_t>(split_cap, std::max<int64_t>(1, tiles_T));
  // more CTAs than SMs: the last ones start a wave late, so every tile goes out
  // by the counter (a static share of theirs would finish a wave late)
  const bool waves = (int64_t)p->n_units * splits > p->n_sms;
  a.static_per = waves ? 0 : tiles_T * kStaticEighths / 8 / splits;
  cudaError_t e = cudaErrorInvalidValue;
  const dim3 grid((unsigned)p->n_units, (unsigned)splits), block((unsigned)((2 * np + 1) * 32));
  switch (p->cfg.v_bits) {
#define GTQ_LAUNCH_VB(VB)                                                                     \
  case VB:                                                                                   \
    if (a.rlen > 0) {                                                                        \
      e = cudaFuncSetAttribute(decode_kernel<VB, true>,                                      \
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);     \
      if (e == cudaSuccess)                                                                  \
        e = launch_pdl(decode_kernel<VB, true>, grid, block, kSmemBytes, s, vmap, a);        \
    } else {                                                                                 \
      e = cudaFuncSetAttribute(decode_kernel<VB, false>,                                     \
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);     \
      if (e == cudaSuccess)                                                                  \
        e = launch_pdl(decode_kernel<VB, false>, grid, block, kSmemBytes, s, vmap, a);       \
    }                                                                                        \
    break;
    GTQ_LAUNCH_VB(0)
    GTQ_LAUNCH_VB(1) GTQ_LAUNCH_VB(2) GTQ_LAUNCH_VB(3) GTQ_LAUNCH_VB(4)
    GTQ_LAUNCH_VB(5) GTQ_LAUNCH_VB(6) GTQ_LAUNCH_VB(7) GTQ_LAUNCH_VB(8)
#undef GTQ_LAUNCH_VB
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace gtq
