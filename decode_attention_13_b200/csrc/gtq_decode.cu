// Fused GQA decode attention over the Block-GTQ packed cache ("RoPE-Aware Bit
// Allocation for KV-Cache Quantization", Abstract: the "packed-cache serving
// path").  No fp16 K or V is materialised: codes are turned into tensor-core
// operands in registers.  One launch per call (decode_kernel), grid = (context
// splits, heads), one CTA per SM:
//   setup   lookup tables, head metadata and M_h^T by bulk copies; after the
//           grid-dependency wait the query heads of the KV head are rotated
//           once, q_rot[pos] = M_h[pos] . q * log2(e) / (sqrt(d) sqrt(m_g)).
//   loop    the split's 64-token tiles, each shared by a pair of warps (32
//           tokens each) and staged by 1-D bulk TMA (cp.async.bulk + mbarrier).
//           Scores: mma.m16n8k16 with A = codebook values of 16 tokens x 16
//           rotated coords and B = q_rot (8 query heads), accumulated per key
//           group and scaled by its fp16 norms; the widest groups use split
//           fp16 (hi/lo) operands.  Online softmax in base 2.  P.V: mma with
//           A = V codebook values (16 dims x 16 tokens) and B = P^T (movmatrix
//           transpose of the score fragment), accumulated in V's rotated basis.
//   merge   the CTA's warps, then the splits: the last CTA of each group of
//           splits merges the group, the last group merges the rest and writes
//           o = R_V^T o_rot / l.
#include <algorithm>
#include <cmath>
#include <cstddef>

#include "gtq_internal.h"

namespace gtq {
namespace {

constexpr int kPairs = 8;  // one CTA per SM: up to 8 warp pairs, 2 tile stages per pair
constexpr int kWarps = 2 * kPairs;
constexpr int kMaxStages = 2;  // tile stages per warp pair
constexpr uint32_t kSuspendHintNs = 1000000;  // mbarrier try_wait suspend-time hint
constexpr uint64_t kWaitNs = 2000000000ull;    // bound of one wait

struct DecodeArgs {
  const uint8_t* packed;
  const HeadMeta* meta;
  const void* q;        // [B][Hq][128] fp16 or fp32 (q_fp32)
  const float* mrow_t;  // [heads][128][128] key rotation, transposed: [dim][packed position]
  const float* rot_v;   // R_V [128][128]
  float* out;           // [B][Hq][128]
  const uint4* dec_image;  // lookup tables (kDecodeImageBytes)
  float* partials;      // [heads][kPartialSlots][8][kPartialStride]
  unsigned* tickets;    // [heads][1 + kMaxMergeGroups] arrival counters of the split merge
  int* status;
  int q_fp32;
  int hkv, gq;
  int64_t T;
  int64_t n_tiles;    // capacity tiles per head
  int tile_bytes;
  int kb, vb;
  int splits;
  int stages;         // tile stages per warp pair
  int area;           // bytes of the stage area
  int rot_off;        // byte offset of the setup scratch in the stage area
  int64_t tiles_T;    // ceil(T / 64)
};

__device__ inline uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ inline void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing bytes on the mbarrier
__device__ inline void bulk_copy(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// L2 policy for the packed cache: streamed once per call, evicted first, so
// that it does not push the tables, rotations and code out of L2
__device__ inline uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// one packed tile: arm the stage's mbarrier with the byte count, then copy
__device__ inline void tile_load(void* dst, const void* src, unsigned bytes, uint64_t* bar,
                                 uint64_t policy) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// bounded wait on an mbarrier phase; returns false after about two seconds.
// Each try suspends the thread until the phase completes or a time hint
// expires, so a waiting warp takes no issue slots from the working ones.
__device__ inline bool mbar_wait(uint64_t* bar, unsigned phase) {
  uint64_t t0 = 0;
  for (unsigned i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase), "r"(kSuspendHintNs)
        : "memory");
    if (ok) return true;
    if ((i & 15u) == 15u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0)
        t0 = now;
      else if (now - t0 > kWaitNs)
        return false;
    }
  }
}

__device__ inline void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ inline uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// programmatic dependent launch: wait for / release the neighbouring grids
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ inline uint32_t pack_half2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// ---------------------------------------------------------------------------
// Code -> fp16 lookups (table layout: gtq_internal.h).  Every lookup address is
// "region offset (an immediate) + (field << k | lane * 4)": one shift and one
// mask-or per lookup.  Widths 1..3 use lane-private pair tables (one lookup per
// half2), widths 4..6 lane-private single-code tables, widths 7..8 and the lo
// parts of narrow split groups one shared single-code table.
// ---------------------------------------------------------------------------

static_assert(sizeof(HeadMeta) % 16 == 0, "metadata is bulk-copied");

struct DecodeSmem {
  uint4 qf[kMaxKt][32];  // per k-tile & lane: hi(slot A), hi(slot B), lo(A), lo(B)
  alignas(16) HeadMeta meta;
  uint2 gdesc[kMaxGroups];  // per key group: 2 width + split | kt0 << 8 | kt1 << 16; byte offset
  uint64_t setup_bar;              // lookup tables and metadata loaded
  uint64_t bar[kPairs][kMaxStages];   // tile loaded (bulk copy complete)
  unsigned done[kPairs][kMaxStages];  // releases of a stage by the two warps of its pair
  float wm[kWarps][8], wl[kWarps][8], wsc[kWarps][8], hm[8], hl[8];
  alignas(16) float qs[8][kD];  // queries of this KV head, then the merged o_rot
  alignas(16) float qr[8][kD];  // rotated, scaled queries
  int flag;
};
// vector (16-byte) and bulk-copy accesses
static_assert(offsetof(DecodeSmem, qf) % 16 == 0 && offsetof(DecodeSmem, meta) % 16 == 0 &&
                  offsetof(DecodeSmem, qs) % 16 == 0 && offsetof(DecodeSmem, qr) % 16 == 0,
              "shared-memory alignment");

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

// Table load from a shared-window address: `addr` already holds the table
// base (8 KB aligned) ORed with the lane and the index; the region offset is
// the load's immediate.
template <uint32_t OFF>
__device__ __forceinline__ uint32_t lds_tab(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(OFF));
  return v;
}

// hi|lo word (fp16 hi in the low half) of the code of width W at bits [P, P + W)
template <int W, int P>
__device__ __forceinline__ uint32_t single_code(const DecodeSmem& s, const uint32_t* x, uint32_t lane4) {
  if constexpr (W >= 4 && W <= 6)
    return lds_tab<kLaneSingleOff(W)>(fld<P, W, 7>(x, lane4));
  else
    return lds_tab<kSharedSingles + kSingleOff(W)>(fld<P, W, 2>(x, lane4 & ~127u));
}

// half2 (hi parts) of codes (2X, 2X + 1), width W, from the bit string x
template <int W, int X>
__device__ __forceinline__ uint32_t pair_hi(const DecodeSmem& s, const uint32_t* x, uint32_t lane4) {
  if constexpr (W <= 3) {
    return lds_tab<kPairOff(W)>(fld<2 * X * W, 2 * W, 7>(x, lane4));
  } else {
    const uint32_t e0 = single_code<W, 2 * X * W>(s, x, lane4);
    const uint32_t e1 = single_code<W, (2 * X + 1) * W>(s, x, lane4);
    return __byte_perm(e0, e1, 0x5410);
  }
}
// hi and lo half2 of codes (2X, 2X + 1) from the single-code tables
template <int W, int X>
__device__ __forceinline__ void pair_hilo(const DecodeSmem& s, const uint32_t* x, uint32_t lane4,
                                          uint32_t& hi, uint32_t& lo) {
  const uint32_t e0 = single_code<W, 2 * X * W>(s, x, lane4);
  const uint32_t e1 = single_code<W, (2 * X + 1) * W>(s, x, lane4);
  hi = __byte_perm(e0, e1, 0x5410);
  lo = __byte_perm(e0, e1, 0x7632);
}

// NB bits of packed codes starting at byte byte_off of tile, realigned to bit 0
// of x[] (x holds NB bits plus up to 24 bits of what follows).
template <int NB>
struct Bits {
  static constexpr int NW = (NB + 31) / 32 + 1;
  uint32_t x[NW];
  __device__ __forceinline__ void load(const uint8_t* tile, int byte_off) {
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(tile + (byte_off & ~3));
    const uint32_t sh = (uint32_t)(byte_off & 3) << 3;
#pragma unroll
    for (int i = 0; i < NW; ++i) x[i] = wp[i];
#pragma unroll
    for (int i = 0; i + 1 < NW; ++i) x[i] = __funnelshift_r(x[i], x[i + 1], sh);
  }
};

// One decode k-tile of a group of width W for this warp's 32 tokens: 8 slots x
// 16 coords; this lane's slots are first + t (A-fragment regs 0/1) and
// first + t + 4 (regs 2/3), its tokens g + 8u for the warp's u = 4h .. 4h + 3,
// i.e. 8W bits of each slot's 16W-bit lane portion.  Slots past the group's
// run read unrelated bits; their q is zero.  When the run has at most 4 slots
// the second half is all padding and is skipped.  SPLIT adds the hi.lo and
// lo.hi terms of the split fp16 product (same accumulator).
template <int W, bool SPLIT>
__device__ __forceinline__ void ktile_step(const DecodeSmem& s, const uint8_t* tile, int koff_a,
                                           bool has_b, uint32_t lane4, const uint4& bq,
                                           float (&C)[2][4]) {
  constexpr bool kCombined = W >= 4;  // single-code tables: hi and lo from one load
  Bits<8 * W> ka, kb;
  ka.load(tile, koff_a);
  if (has_b) kb.load(tile, koff_a + 64 * W);
#define GTQ_MT(MT)                                                                   \
  {                                                                                  \
    uint32_t ah[4], al[4];                                                           \
    if constexpr (kCombined) {                                                       \
      pair_hilo<W, 2 * (MT)>(s, ka.x, lane4, ah[0], al[0]);                          \
      pair_hilo<W, 2 * (MT) + 1>(s, ka.x, lane4, ah[1], al[1]);                      \
      if (has_b) {                                                                   \
        pair_hilo<W, 2 * (MT)>(s, kb.x, lane4, ah[2], al[2]);                        \
        pair_hilo<W, 2 * (MT) + 1>(s, kb.x, lane4, ah[3], al[3]);                    \
      } else {                                                                       \
        ah[2] = ah[3] = al[2] = al[3] = 0u;                                          \
      }                                                                              \
    } else {                                                                         \
      ah[0] = pair_hi<W, 2 * (MT)>(s, ka.x, lane4);                                  \
      ah[1] = pair_hi<W, 2 * (MT) + 1>(s, ka.x, lane4);                              \
      ah[2] = has_b ? pair_hi<W, 2 * (MT)>(s, kb.x, lane4) : 0u;                     \
      ah[3] = has_b ? pair_hi<W, 2 * (MT) + 1>(s, kb.x, lane4) : 0u;                 \
      if constexpr (SPLIT) {                                                         \
        uint32_t dummy;                                                              \
        pair_hilo<W, 2 * (MT)>(s, ka.x, lane4, dummy, al[0]);                        \
        pair_hilo<W, 2 * (MT) + 1>(s, ka.x, lane4, dummy, al[1]);                    \
        al[2] = al[3] = 0u;                                                          \
        if (has_b) {                                                                 \
          pair_hilo<W, 2 * (MT)>(s, kb.x, lane4, dummy, al[2]);                      \
          pair_hilo<W, 2 * (MT) + 1>(s, kb.x, lane4, dummy, al[3]);                  \
        }                                                                            \
      }                                                                              \
    }                                                                                \
    mma16816(C[MT], ah, bq.x, bq.y);                                                 \
    if constexpr (SPLIT) {                                                           \
      mma16816(C[MT], ah, bq.z, bq.w);                                               \
      mma16816(C[MT], al, bq.x, bq.y);                                               \
    }                                                                                \
  }
  GTQ_MT(0) GTQ_MT(1)
#undef GTQ_MT
}

template <int W, bool SPLIT>
__device__ __forceinline__ void group_scores(const DecodeSmem& s, const uint8_t* tile, uint2 desc,
                                             int koff_lane, uint32_t lane4, int lane,
                                             float (&C)[2][4]) {
  const int kt0 = (desc.x >> 8) & 0xff, kt1 = (desc.x >> 16) & 0xff;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int r = 0; r < 4; ++r) C[mt][r] = 0.f;
#pragma unroll 1
  for (int kt = kt0; kt < kt1; ++kt)
    ktile_step<W, SPLIT>(s, tile, koff_lane + (kt - kt0) * 128 * W, s.meta.kt_nslots[kt] > 4,
                         lane4, s.qf[kt][lane], C);
}

// P.V for one dim tile and this warp's 32 tokens: 16 codes of width VB per lane
// (pairs 8h .. 8h + 7 of the lane's 32-code portion), 2 token k-tiles
template <int VB>
__device__ __forceinline__ void value_tile(const DecodeSmem& s, const uint8_t* lane_codes, int h,
                                           uint32_t lane4, const uint32_t (&PB)[2][2],
                                           float (&o)[4]) {
  Bits<16 * VB> v;
  v.load(lane_codes, 2 * VB * h);
#define GTQ_V_KTILE(KK)                                                            \
  {                                                                                \
    const uint32_t av[4] = {pair_hi<VB, 4 * (KK)>(s, v.x, lane4),                  \
                            pair_hi<VB, 4 * (KK) + 1>(s, v.x, lane4),              \
                            pair_hi<VB, 4 * (KK) + 2>(s, v.x, lane4),              \
                            pair_hi<VB, 4 * (KK) + 3>(s, v.x, lane4)};             \
    mma16816(o, av, PB[KK][0], PB[KK][1]);                                         \
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
// as a partial to dst (global) or, normalised (o / L), to o_rot (shared).
// Work item = (query head, parity of j) per warp, lane = 4 dims: a warp reads
// whole partial rows (coalesced), all of its up to 8 partials in flight at
// once; the two parities combine through `scratch` (shared, 2 x 8 x
// kPartialStride floats).  Partials come from other CTAs: loads bypass L1.
__device__ __noinline__ void merge_partials(const float* head_parts, int first, int count,
                                            float* dst, float (*o_rot)[kD], float* scratch) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int item = warp; item < 16; item += nwarps) {
    const int hh = item >> 1, sub = item & 1;
    float2 ml[kMergeGroup / 2];
    float4 oj[kMergeGroup / 2];
#pragma unroll
    for (int b = 0; b < kMergeGroup / 2; ++b) {
      const int j = sub + 2 * b;
      ml[b] = make_float2(-1e30f, 0.f);
      oj[b] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < count) {
        const float* pj = head_parts + ((size_t)(first + j) * 8 + hh) * kPartialStride;
        ml[b] = __ldcg(reinterpret_cast<const float2*>(pj));
        oj[b] = __ldcg(reinterpret_cast<const float4*>(pj + 4) + lane);
      }
    }
    float M = ml[0].x;
#pragma unroll
    for (int b = 1; b < kMergeGroup / 2; ++b) M = fmaxf(M, ml[b].x);
    float L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int b = 0; b < kMergeGroup / 2; ++b) {
      const float w = exp2f(ml[b].x - M);
      L = fmaf(w, ml[b].y, L);
      o.x = fmaf(w, oj[b].x, o.x);
      o.y = fmaf(w, oj[b].y, o.y);
      o.z = fmaf(w, oj[b].z, o.z);
      o.w = fmaf(w, oj[b].w, o.w);
    }
    float* sc = scratch + (size_t)(sub * 8 + hh) * kPartialStride;
    reinterpret_cast<float4*>(sc + 4)[lane] = o;
    if (lane == 0) *reinterpret_cast<float2*>(sc) = make_float2(M, L);
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 8 * 32; idx += blockDim.x) {
    const int hh = idx >> 5, d4 = idx & 31;
    const float* s0 = scratch + (size_t)hh * kPartialStride;
    const float* s1 = scratch + (size_t)(8 + hh) * kPartialStride;
    const float2 ml0 = *reinterpret_cast<const float2*>(s0), ml1 = *reinterpret_cast<const float2*>(s1);
    const float4 o0 = reinterpret_cast<const float4*>(s0 + 4)[d4];
    const float4 o1 = reinterpret_cast<const float4*>(s1 + 4)[d4];
    const float M = fmaxf(ml0.x, ml1.x), w0 = exp2f(ml0.x - M), w1 = exp2f(ml1.x - M);
    const float L = w0 * ml0.y + w1 * ml1.y;
    const float4 o = make_float4(w0 * o0.x + w1 * o1.x, w0 * o0.y + w1 * o1.y, w0 * o0.z + w1 * o1.z,
                                 w0 * o0.w + w1 * o1.w);
    if (dst) {
      float* pd = dst + hh * kPartialStride;
      reinterpret_cast<float4*>(pd + 4)[d4] = o;
      if (d4 == 0) *reinterpret_cast<float2*>(pd) = make_float2(M, L);
    } else {
      const float inv = 1.f / L;
      *reinterpret_cast<float4*>(&o_rot[hh][4 * d4]) = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    }
  }
}

template <int VB>
__global__ void __launch_bounds__(kWarps * 32, 1) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem& s = *reinterpret_cast<DecodeSmem*>(smem_raw);
  const size_t stage_off = (sizeof(DecodeSmem) + 127) & ~size_t(127);
  const int stride = (a.tile_bytes + 127) & ~127;
  const int head = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int nw = blockDim.x >> 5;  // warps in this CTA (even, <= kWarps)
  const int np = nw >> 1;          // warp pairs: both warps of a pair share one tile
  const int pair = warp >> 1, wh = warp & 1;  // this warp: tokens 32 wh .. 32 wh + 31

  // Shared memory after DecodeSmem: tile stages, stage-major (stage st of pair
  // p at (st * np + p) * stride); at setup the transposed key rotation M_h^T
  // and the rotation's partial sums sit at a.rot_off, inside stages >= 1, whose
  // tiles load once the rotation is done.
  const int stages = a.stages;
  uint8_t* stage_base = smem_raw + stage_off;
  auto stage_ptr = [&](int st) { return stage_base + (size_t)(st * np + pair) * stride; };
  float* mt = reinterpret_cast<float*>(stage_base + a.rot_off);  // M_h^T [dim][pos]
  float* rot_part = mt + kD * kD;                                 // [4][8][128]
  float(*qt)[8] = reinterpret_cast<float(*)[8]>(&s.qs[0][0]);    // q^T [dim][head]

  // lookup tables after the stage area, at an 8 KB-aligned shared address (so
  // that table base, index and lane combine by OR)
  const uint32_t raw_sa = smem_u32(smem_raw);
  const uint32_t tab_sa = (raw_sa + (uint32_t)(stage_off + a.area) + 8191u) & ~8191u;
  uint8_t* tab = smem_raw + (tab_sa - raw_sa);

  // Setup: lookup tables, head metadata and M_h^T by bulk copies (issued
  // first: nothing here depends on the previous grid), then stage 0 of every
  // pair; the queries follow the grid-dependency wait.
  if (tid == 0) {
    mbar_init(&s.setup_bar, 1);
    for (int p = 0; p < np; ++p)
      for (int st = 0; st < stages; ++st) {
        mbar_init(&s.bar[p][st], 1);
        s.done[p][st] = 0u;
      }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(&s.setup_bar)),
                 "r"((unsigned)(kDecodeImageBytes + sizeof(HeadMeta) + kD * kD * sizeof(float)))
                 : "memory");
    bulk_copy(tab, a.dec_image, kDecodeImageBytes, &s.setup_bar);
    bulk_copy(&s.meta, a.meta + head, sizeof(HeadMeta), &s.setup_bar);
    bulk_copy(mt, a.mrow_t + (size_t)head * kD * kD, kD * kD * sizeof(float), &s.setup_bar);
  }
  __syncthreads();  // barrier initialisation visible
  pdl_launch_dependents();
  bool failed = __syncthreads_or(!mbar_wait(&s.setup_bar, 0));
  const HeadMeta& m = s.meta;
  const int load_bytes = 1024 * (a.kb + VB) + 128 + 128 * m.n_groups;
  const int knorm_off = 1024 * (a.kb + VB) + 128, vnorm_off = 1024 * (a.kb + VB);
  // lookup-table base | lane * 4: the high bits of every table address
  const uint32_t lane4 = tab_sa | ((uint32_t)lane << 2);

  // tiles of this split, dealt to warp pairs round-robin
  const int64_t per = (a.tiles_T + a.splits - 1) / a.splits;
  const int64_t tb0 = (int64_t)split * per, tb1 = failed ? tb0 : min(a.tiles_T, tb0 + per);
  const uint8_t* head_base = a.packed + (size_t)head * a.n_tiles * a.tile_bytes;
  const uint64_t stream_pol = evict_first_policy();
  auto first_loads = [&](int st0, int st1) {
    if (wh == 0 && lane == 0 && !failed) {
      for (int st = st0; st < st1; ++st) {
        const int64_t tile = tb0 + pair + (int64_t)np * st;
        if (tile < tb1) tile_load(stage_ptr(st), head_base + (size_t)tile * a.tile_bytes,
                                  (unsigned)load_bytes, &s.bar[pair][st], stream_pol);
      }
    }
  };
  first_loads(0, 1);
  pdl_wait();  // the queries may come from the previous grid
  {
    const int b = head / a.hkv, h = head % a.hkv;
    for (int i = tid; i < 8 * kD; i += blockDim.x) {
      const int hh = i >> 7, d = i & (kD - 1);
      float v = 0.f;
      if (hh < a.gq) {
        const size_t qi = ((size_t)b * a.hkv * a.gq + (size_t)h * a.gq + hh) * kD + d;
        v = a.q_fp32 ? reinterpret_cast<const float*>(a.q)[qi]
                     : __half2float(reinterpret_cast<const __half*>(a.q)[qi]);
      }
      qt[d][hh] = v;
    }
  }
  __syncthreads();
  // q_rot[hh][pos] = M_h[pos] . q[hh] * log2(e) / (sqrt(d) sqrt(m_g)).  Task = (pos,
  // quarter of d): a warp holds 32 consecutive positions of one quarter, so the
  // M_h^T reads are contiguous and the q reads broadcasts.
  for (int task = tid; task < 4 * kD; task += blockDim.x) {
    const int pos = task & (kD - 1), qd = task >> 7;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int i = 0; i < 32; ++i) {
      const int d = 32 * qd + i;
      const float mv = mt[d * kD + pos];
      const float4 qa = *reinterpret_cast<const float4*>(&qt[d][0]);
      const float4 qb = *reinterpret_cast<const float4*>(&qt[d][4]);
      acc[0] = fmaf(mv, qa.x, acc[0]);
      acc[1] = fmaf(mv, qa.y, acc[1]);
      acc[2] = fmaf(mv, qa.z, acc[2]);
      acc[3] = fmaf(mv, qa.w, acc[3]);
      acc[4] = fmaf(mv, qb.x, acc[4]);
      acc[5] = fmaf(mv, qb.y, acc[5]);
      acc[6] = fmaf(mv, qb.z, acc[6]);
      acc[7] = fmaf(mv, qb.w, acc[7]);
    }
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) rot_part[(qd * 8 + hh) * kD + pos] = acc[hh];
  }
  __syncthreads();
  for (int i = tid; i < 8 * kD; i += blockDim.x) {
    const int hh = i >> 7, pos = i & (kD - 1), slot = pos >> 1;
    // base-2 logits: log2(e) / sqrt(128), and 1/sqrt(m_g) of the group
    const float sc = slot < m.n_slots ? m.inv_sqrt_m[m.slot_group[slot]] *
                                            (1.4426950408889634f * 0.08838834764831845f)
                                      : 0.f;
    s.qr[hh][pos] = ((rot_part[hh * kD + pos] + rot_part[(8 + hh) * kD + pos]) +
                     (rot_part[(16 + hh) * kD + pos] + rot_part[(24 + hh) * kD + pos])) * sc;
  }
  __syncthreads();  // M_h^T and the partial sums are dead: stages >= 1 may load
  if (wh == 0 && lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  first_loads(1, stages);
  if (tid < m.n_groups) {
    const int gi = tid;
    s.gdesc[gi] = make_uint2((2u * m.grp_width[gi] + (m.grp_split[gi] & 1u)) |
                                 ((uint32_t)m.grp_kt0[gi] << 8) | ((uint32_t)m.grp_kt1[gi] << 16),
                             (uint32_t)m.slot_koff[m.grp_first_slot[gi]]);
  }
  // B fragments (query) of every decode k-tile; slots past the k-tile's run are zero
  for (int idx = tid; idx < m.n_ktiles * 32; idx += blockDim.x) {
    const int kt = idx >> 5, ln = idx & 31, gg = ln >> 2, tt = ln & 3;
    uint32_t outv[4];
    for (int half = 0; half < 2; ++half) {
      const int sl = tt + 4 * half;  // slot within the k-tile
      const bool in = sl < m.kt_nslots[kt];
      const int pos = 2 * (m.kt_first_slot[kt] + sl);
      const float v0 = in ? s.qr[gg][pos] : 0.f, v1 = in ? s.qr[gg][pos + 1] : 0.f;
      const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
      outv[half] = pack_half2(h0, h1);
      outv[2 + half] = pack_half2(__float2half_rn(v0 - __half2float(h0)),
                                  __float2half_rn(v1 - __half2float(h1)));
    }
    s.qf[kt][ln] = make_uint4(outv[0], outv[1], outv[2], outv[3]);
  }
  __syncthreads();

  float mrun[2] = {-1e30f, -1e30f}, lrun[2] = {0.f, 0.f};
  float O[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) O[i][0] = O[i][1] = O[i][2] = O[i][3] = 0.f;

  int it = 0, st = 0;
  unsigned phase = 0u;
  for (int64_t tile = tb0 + pair; tile < tb1; tile += np, ++it) {
    if (!mbar_wait(&s.bar[pair][st], phase)) {
      failed = true;
      break;
    }
    const uint8_t* tl = stage_ptr(st);

    // ------------------------------------------------------------ scores
    float S[2][4], C[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) S[mt][r] = 0.f;
#pragma unroll 1
    for (int gi = 0; gi < m.n_groups; ++gi) {
      // group descriptor: 2 width + split | kt0 << 8 | kt1 << 16, first slot's byte offset
      const uint2 desc = s.gdesc[gi];
      const int W = (desc.x >> 1) & 0xf;
      // lane portion of slot t: 16W bits at byte 16W t + 2W g; this warp's half: + W wh
      const int koff_lane = (int)desc.y + W * (16 * t + 2 * g + wh);
      switch (desc.x & 0x1f) {  // 2 W + split
#define GTQ_GROUP(WW)                                                          \
  case 2 * WW:                                                                 \
    group_scores<WW, false>(s, tl, desc, koff_lane, lane4, lane, C);           \
    break;                                                                     \
  case 2 * WW + 1:                                                             \
    group_scores<WW, true>(s, tl, desc, koff_lane, lane4, lane, C);            \
    break;
        GTQ_GROUP(1) GTQ_GROUP(2) GTQ_GROUP(3) GTQ_GROUP(4)
        GTQ_GROUP(5) GTQ_GROUP(6) GTQ_GROUP(7) GTQ_GROUP(8)
#undef GTQ_GROUP
        default: break;
      }
      // group complete: scale by its fp16 norms (tokens g + 8u, u = 4wh .. 4wh + 3)
      const uint2 nq = *reinterpret_cast<const uint2*>(tl + knorm_off + gi * 128 + g * 16 + wh * 8);
      const __half2* nh = reinterpret_cast<const __half2*>(&nq);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const float2 n = __half22float2(nh[mt]);
        S[mt][0] = fmaf(n.x, C[mt][0], S[mt][0]);
        S[mt][1] = fmaf(n.x, C[mt][1], S[mt][1]);
        S[mt][2] = fmaf(n.y, C[mt][2], S[mt][2]);
        S[mt][3] = fmaf(n.y, C[mt][3], S[mt][3]);
      }
    }
    // ------------------------------------------------------ online softmax
    const int64_t tok0 = tile * kTile + 32 * wh;
    const bool full = tok0 + 32 <= a.T;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = 16 * mt + g + 8 * (r >> 1);
        if (!full && tok0 + j >= a.T) S[mt][r] = -INFINITY;
        mx[r & 1] = fmaxf(mx[r & 1], S[mt][r]);
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
    const uint2 vq = *reinterpret_cast<const uint2*>(tl + vnorm_off + g * 16 + wh * 8);
    const __half2* vnh = reinterpret_cast<const __half2*>(&vq);
    uint32_t PB[2][2];
    const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      float2 vn = __half22float2(vnh[mt]);
      vn.x *= inv_sqrt_d;
      vn.y *= inv_sqrt_d;
      float pp[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = 16 * mt + g + 8 * (r >> 1);
        const float p = exp2f(S[mt][r] - mrun[r & 1]);
        lrun[r & 1] += p;
        const float nv = (r >> 1) ? vn.y : vn.x;
        pp[r] = (full || tok0 + j < a.T) ? p * nv : 0.f;
      }
      PB[mt][0] = movmatrix_t(pack_half2(__float2half_rn(pp[0]), __float2half_rn(pp[1])));
      PB[mt][1] = movmatrix_t(pack_half2(__float2half_rn(pp[2]), __float2half_rn(pp[3])));
    }
    // ---------------------------------------------------------------- P.V
    const uint8_t* vcodes = tl + 1024 * a.kb;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      value_tile<VB>(s, vcodes + ((i * 8 + g) * 4 + t) * VB * 4, wh, lane4, PB, O[i]);
    // ------------------------------------- release the stage; the second warp
    // of the pair to release it refills it
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const unsigned prev = atomicAdd(&s.done[pair][st], 1u);
      if (prev & 1u) {
        __threadfence_block();
        const int64_t nxt = tile + (int64_t)np * stages;
        if (nxt < tb1) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          tile_load(stage_ptr(st), head_base + (size_t)nxt * a.tile_bytes, (unsigned)load_bytes,
                    &s.bar[pair][st], stream_pol);
        }
      }
    }
    if (++st == stages) {
      st = 0;
      phase ^= 1u;
    }
  }
  if (failed && lane == 0) atomicOr(a.status, kStatusTimeout);

  // ------------------------------------------------- merge the warps in the CTA
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 4);
    lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 8);
    lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 16);
  }
  __syncthreads();  // every warp is done with its stages: reuse them for R_V and o
  // R_V is staged in every CTA (only the one that finishes the merge uses it;
  // the copy is in flight meanwhile, and every CTA waits for it before exit)
  float* rv = reinterpret_cast<float*>(stage_base);            // R_V [128][128]
  float* wo = reinterpret_cast<float*>(stage_base) + kD * kD;  // [warp][8][128]
  if (tid == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(&s.setup_bar)),
                 "r"((unsigned)(kD * kD * sizeof(float)))
                 : "memory");
    bulk_copy(rv, a.rot_v, kD * kD * sizeof(float), &s.setup_bar);
  }
  if (g == 0) {
    s.wm[warp][2 * t] = mrun[0];
    s.wm[warp][2 * t + 1] = mrun[1];
    s.wl[warp][2 * t] = lrun[0];
    s.wl[warp][2 * t + 1] = lrun[1];
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float* o = wo + warp * 8 * kD;
    o[(2 * t) * kD + 16 * i + g] = O[i][0];
    o[(2 * t + 1) * kD + 16 * i + g] = O[i][1];
    o[(2 * t) * kD + 16 * i + g + 8] = O[i][2];
    o[(2 * t + 1) * kD + 16 * i + g + 8] = O[i][3];
  }
  __syncthreads();
  if (tid < 8) {  // per query head: max over the warps, their scales and the sum of l
    const int hh = tid;
    float M = -1e30f;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, s.wm[w][hh]);
    float L = 0.f;
    for (int w = 0; w < nw; ++w) {
      const float sc = exp2f(s.wm[w][hh] - M);
      s.wsc[w][hh] = sc;
      L = fmaf(sc, s.wl[w][hh], L);
    }
    s.hm[hh] = M;
    s.hl[hh] = L;
  }
  __syncthreads();
  const int S = a.splits;
  float* head_parts = a.partials + (size_t)head * kPartialSlots * 8 * kPartialStride;
  float* part = head_parts + (size_t)split * 8 * kPartialStride;
  // this CTA's (m, l, o_rot): the output itself with a single split, else its
  // partial in global memory
  for (int idx = tid; idx < 8 * kD; idx += blockDim.x) {
    const int hh = idx >> 7, d = idx & (kD - 1);
    float v = 0.f;
    for (int w = 0; w < nw; ++w) v = fmaf(s.wsc[w][hh], wo[(w * 8 + hh) * kD + d], v);
    if (S == 1) {
      s.qs[hh][d] = v / s.hl[hh];
    } else {
      part[hh * kPartialStride + 4 + d] = v;
      if (d == 0) *reinterpret_cast<float2*>(part + hh * kPartialStride) = make_float2(s.hm[hh], s.hl[hh]);
    }
  }
  // ---------------- merge of the splits, without waiting: the last CTA to
  // arrive in a group of kMergeGroup splits merges the group into a
  // second-level partial, and the last group to finish merges those.  Arrival
  // order comes from per-head tickets (acquire-release atomics); the last
  // arriver resets its ticket for the next call.
  float* mscratch = wo;  // the warps' o are consumed: merge scratch
  bool finish = S == 1;
  if (!finish) {
    unsigned* tickets = a.tickets + (size_t)head * (1 + kMaxMergeGroups);
    const int n_groups = (S + kMergeGroup - 1) / kMergeGroup;
    const int grp = split / kMergeGroup;
    const int n1 = min(kMergeGroup, S - grp * kMergeGroup);
    if (arrive_last(&tickets[1 + grp], (unsigned)n1, &s.flag)) {
      if (n_groups == 1) {
        merge_partials(head_parts, grp * kMergeGroup, n1, nullptr, s.qs, mscratch);
        finish = true;
      } else {
        merge_partials(head_parts, grp * kMergeGroup, n1,
                       head_parts + (size_t)(kMaxSplits + grp) * 8 * kPartialStride, nullptr,
                       mscratch);
        if (arrive_last(&tickets[0], (unsigned)n_groups, &s.flag)) {
          merge_partials(head_parts, kMaxSplits, n_groups, nullptr, s.qs, mscratch);
          finish = true;
        }
      }
    }
  }
  const bool rv_ok = mbar_wait(&s.setup_bar, 1);  // no CTA exits with the copy in flight
  if (!finish) return;
  if (!rv_ok) {
    if (tid == 0) atomicOr(a.status, kStatusTimeout);
    return;
  }
  __syncthreads();
  // out[hh][dd] = sum_r R_V[r][dd] o_rot[hh][r]
  {
    const int b = head / a.hkv, h = head % a.hkv;
    float* out_head = a.out + ((size_t)b * a.hkv * a.gq + (size_t)h * a.gq) * kD;
    for (int idx = tid; idx < 8 * (kD / 2); idx += blockDim.x) {
      const int hh = idx / (kD / 2), dd = 2 * (idx % (kD / 2));
      if (hh >= a.gq) continue;
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
      for (int r = 0; r < kD; ++r) {
        const float2 w = *reinterpret_cast<const float2*>(rv + r * kD + dd);
        const float o = s.qs[hh][r];
        acc0 = fmaf(w.x, o, acc0);
        acc1 = fmaf(w.y, o, acc1);
      }
      *reinterpret_cast<float2*>(out_head + hh * kD + dd) = make_float2(acc0, acc1);
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
                          int q_dtype, float* out, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  DecodeArgs a;
  a.packed = packed;
  a.meta = p->d_meta;
  a.q = q;
  a.q_fp32 = q_dtype == GTQ_DTYPE_FP32;
  a.mrow_t = p->d_mrow_t;
  a.rot_v = p->tab.rot_v;
  a.out = out;
  a.tickets = p->d_tickets;
  a.hkv = p->cfg.n_kv_heads;
  a.gq = p->g_q;
  a.dec_image = p->tab.dec_image;
  a.partials = p->d_partials;
  a.status = p->d_status;
  a.T = T;
  a.n_tiles = p->n_tiles;
  a.tile_bytes = (int)p->tile_bytes;
  a.kb = p->cfg.k_bits;
  a.vb = p->cfg.v_bits;
  a.tiles_T = (T + kTile - 1) / kTile;
  const size_t stage_off = (sizeof(DecodeSmem) + 127) & ~size_t(127);
  const size_t stride = (p->tile_bytes + 127) & ~size_t(127);
  int dev_smem = 0;
  cudaDeviceGetAttribute(&dev_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, p->device);
  // Stage area: the tile stages (two per pair, as many pairs as fit); at the
  // end R_V, the warps' o and the merge scratch; at setup, the setup scratch
  // (M_h^T and the rotation's partial sums) at its top, clear of stage 0.
  constexpr size_t kSetupScratch = (size_t)kD * kD * 4 + (size_t)4 * 8 * kD * 4;
  auto area_for = [&](int np_, int st_) {
    return std::max({stride * np_ * st_, (size_t)kD * kD * 4 + (size_t)2 * np_ * 8 * kD * 4,
                     stride * np_ + kSetupScratch});
  };
  constexpr size_t kTables = (size_t)kDecodeImageBytes + 8192;  // + alignment slack
  const int stages = kMaxStages;
  int np = kPairs;
  while (np > 1 && stage_off + area_for(np, stages) + kTables > (size_t)dev_smem) --np;
  if (stage_off + area_for(np, stages) + kTables > (size_t)dev_smem) return cudaErrorInvalidValue;
  a.stages = stages;
  const int nw = 2 * np;
  const size_t area = area_for(np, stages);
  a.rot_off = (int)(area - kSetupScratch);
  a.area = (int)area;
  const size_t smem = stage_off + area + kTables;
  int per_sm = 1;
  switch (a.vb) {
#define GTQ_OCC_VB(VB)                                                                           \
  case VB:                                                                                     \
    cudaFuncSetAttribute(decode_kernel<VB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<VB>, nw * 32, smem); \
    break;
    GTQ_OCC_VB(1) GTQ_OCC_VB(2) GTQ_OCC_VB(3) GTQ_OCC_VB(4)
    GTQ_OCC_VB(5) GTQ_OCC_VB(6) GTQ_OCC_VB(7) GTQ_OCC_VB(8)
#undef GTQ_OCC_VB
  }
  // one wave of resident CTAs: the split merge waits for every CTA of a head
  const int capacity = std::max(1, per_sm) * p->n_sms;
  int splits = std::max(1, capacity / p->n_heads);
  splits = (int)std::min<int64_t>(splits, (a.tiles_T + np - 1) / np);
  splits = std::max(1, std::min(splits, kMaxSplits));
  // every split must own at least one tile
  const int64_t per = (a.tiles_T + splits - 1) / splits;
  splits = (int)((a.tiles_T + per - 1) / per);
  a.splits = splits;
  e = cudaErrorInvalidValue;
  switch (a.vb) {
#define GTQ_LAUNCH_VB(VB)                                                                       \
  case VB:                                                                                     \
    e = cudaFuncSetAttribute(decode_kernel<VB>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                             (int)smem);                                                        \
    if (e == cudaSuccess)                                                                      \
      e = launch_pdl(decode_kernel<VB>, dim3(splits, p->n_heads), dim3(nw * 32), smem, s, a);  \
    break;
    GTQ_LAUNCH_VB(1) GTQ_LAUNCH_VB(2) GTQ_LAUNCH_VB(3) GTQ_LAUNCH_VB(4)
    GTQ_LAUNCH_VB(5) GTQ_LAUNCH_VB(6) GTQ_LAUNCH_VB(7) GTQ_LAUNCH_VB(8)
#undef GTQ_LAUNCH_VB
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace gtq
