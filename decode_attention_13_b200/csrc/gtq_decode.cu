// Fused GQA decode attention over the Block-GTQ packed cache ("RoPE-Aware Bit
// Allocation for KV-Cache Quantization", Abstract: the "packed-cache serving
// path").  No fp16 K or V is materialised: codes are turned into tensor-core
// operands in registers.
//
//   rotate_q_kernel  q_rot[pos] = M_h[pos] . q * log2(e) / (sqrt(d) sqrt(m_g)):
//                    every query head of a KV head rotated once per call.
//   decode_kernel    split-K over the context.  A warp owns 64-token tiles
//                    staged by 1-D bulk TMA (cp.async.bulk + mbarrier).  Scores:
//                    mma.m16n8k16 with A = codebook values of 16 tokens x 16
//                    rotated coords and B = q_rot (8 query heads), accumulated
//                    per group and scaled by the fp16 group norms; the widest
//                    groups use split fp16 (hi/lo) operands.  Online softmax in
//                    base 2.  P.V: mma with A = V codebook values (16 dims x 16
//                    tokens) and B = P^T (movmatrix transpose of the score
//                    fragment), accumulated in V's rotated basis.
//   merge_kernel     merge of the split partials (m, l, o) per query head and
//                    o = R_V^T o_rot / l.
#include <algorithm>
#include <cmath>
#include <cstddef>

#include "gtq_internal.h"

namespace gtq {
namespace {

constexpr int kWarps = 12;  // one CTA per SM: up to 12 warps, 2 private tile stages each
constexpr int kStages = 2;
constexpr unsigned kSpinLimit = 1u << 26;
constexpr unsigned kBarrierSpinLimit = 1u << 24;  // x >= 64 ns: over a second

struct DecodeArgs {
  const uint8_t* packed;
  const HeadMeta* meta;
  const void* q;        // [B][Hq][128] fp16 or fp32 (q_fp32)
  const float* mrow;    // [heads][128][128] key rotation rows in packed order
  const float* rot_v;   // R_V [128][128]
  float* out;           // [B][Hq][128]
  const uint4* dec_image;  // lookup tables (kDecodeImageBytes)
  float* partials;      // [heads][kPartialSlots][8][kPartialStride]
  unsigned* tickets;    // [heads][1 + kMaxMergeGroups]
  int* status;
  int q_fp32;
  int hkv, gq;
  int64_t T;
  int64_t n_tiles;    // capacity tiles per head
  int tile_bytes;
  int kb, vb;
  int splits;
  int64_t tiles_T;    // ceil(T / 64)
};

__device__ inline uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ inline void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ inline void bulk_load(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// bounded wait on an mbarrier phase; returns false if the bound expired
__device__ inline bool mbar_wait(uint64_t* bar, unsigned phase) {
  for (unsigned i = 0; i < kSpinLimit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    if (ok) return true;
  }
  return false;
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
// Code -> fp16 lookups.
//
// Pair tables (widths 1..3, fp16 hi parts): entry idx = c0 | c1 << w holds the
// half2 (cb[c0], cb[c1]); every lane has its own copy (word idx * 32 + lane), so
// a warp-wide lookup never has a bank conflict.  Width w's table sits at byte
// offset kPairOff(w), chosen so that offset | idx * 128 | lane * 4 needs no add.
// Single-code tables (widths 1..8, 2^w entries of 32 bits: fp16 hi part in the
// low half, fp16 lo part in the high half): at byte offset 2048 - 2^(w+3) inside
// a 2 KB region, so offset | code * 4 needs no add; widths up to 5 occupy at
// most 32 banks and never conflict.
// ---------------------------------------------------------------------------

struct DecodeSmem {
  uint32_t pair[kPairBytes / 4];  // pair and single tables: one contiguous image
  uint32_t single[kSingleBytes / 4];
  uint4 qf[kMaxKt][32];  // per k-tile & lane: hi(slot A), hi(slot B), lo(A), lo(B)
  HeadMeta meta;
  uint64_t bar[kWarps][kStages];
  float wm[kWarps][8], wl[kWarps][8], wsc[kWarps][8], hm[8], hl[8];
  float qs[8][kD];  // queries of this KV head, then the merged o_rot
  float qr[8][kD];  // rotated, scaled queries
  int flag;
};

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

__device__ __forceinline__ uint32_t lds32(const DecodeSmem& s, uint32_t byte_off) {
  return *reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(s.pair) + byte_off);
}
__device__ __forceinline__ uint32_t lds_single(const DecodeSmem& s, uint32_t byte_off) {
  return *reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(s.single) + byte_off);
}

// half2 of codes (2x, 2x+1), width W, from the bit string x (pair at bits [2xW, 2xW + 2W))
template <int W, int X>
__device__ __forceinline__ uint32_t pair_hi(const DecodeSmem& s, const uint32_t* x, uint32_t lane_pair) {
  if constexpr (W <= 3) {
    return lds32(s, fld<2 * X * W, 2 * W, 7>(x, lane_pair));
  } else {
    const uint32_t e0 = lds_single(s, fld<2 * X * W, W, 2>(x, kSingleOff(W)));
    const uint32_t e1 = lds_single(s, fld<(2 * X + 1) * W, W, 2>(x, kSingleOff(W)));
    return __byte_perm(e0, e1, 0x5410);
  }
}
// hi and lo half2 of codes (2x, 2x+1) from the combined single-code table
template <int W, int X>
__device__ __forceinline__ void pair_hilo(const DecodeSmem& s, const uint32_t* x, uint32_t& hi,
                                          uint32_t& lo) {
  const uint32_t e0 = lds_single(s, fld<2 * X * W, W, 2>(x, kSingleOff(W)));
  const uint32_t e1 = lds_single(s, fld<(2 * X + 1) * W, W, 2>(x, kSingleOff(W)));
  hi = __byte_perm(e0, e1, 0x5410);
  lo = __byte_perm(e0, e1, 0x7632);
}

// The 16w-bit portion of one key slot for this lane (tokens g + 8u, u = 0..7),
// realigned to bit 0 of x[] (portions start at an even byte).
template <int W>
struct KeyWords {
  static constexpr int NW = (16 * W + 31) / 32 + 1;
  uint32_t x[NW];
  __device__ __forceinline__ void load(const uint8_t* tile, int byte_off) {
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(tile + (byte_off & ~3));
    const uint32_t sh = (byte_off & 2) << 3;  // 0 or 16
#pragma unroll
    for (int i = 0; i < NW; ++i) x[i] = wp[i];
#pragma unroll
    for (int i = 0; i + 1 < NW; ++i) x[i] = __funnelshift_r(x[i], x[i + 1], sh);
  }
};

// One decode k-tile of a group of width W: 8 slots x 16 coords; this lane's
// slots are first + t (A-fragment regs 0/1) and first + t + 4 (regs 2/3).
// Slots past the group's run read unrelated bits; their q is zero.  When the
// run has at most 4 slots the second half is all padding and is skipped.
// SPLIT adds the hi.lo and lo.hi terms of the split fp16 product (same accumulator).
template <int W, bool SPLIT>
__device__ __forceinline__ void ktile_step(const DecodeSmem& s, const uint8_t* tile, int koff_a,
                                           bool has_b, uint32_t lane_pair, const uint4& bq,
                                           float (&C)[4][4]) {
  constexpr bool kCombined = W >= 4;  // single-code table: hi and lo from one load
  KeyWords<W> ka, kb;
  ka.load(tile, koff_a);
  if (has_b) kb.load(tile, koff_a + 64 * W);
#define GTQ_MT(MT)                                                                   \
  {                                                                                  \
    uint32_t ah[4], al[4];                                                           \
    if constexpr (kCombined) {                                                       \
      pair_hilo<W, 2 * (MT)>(s, ka.x, ah[0], al[0]);                                 \
      pair_hilo<W, 2 * (MT) + 1>(s, ka.x, ah[1], al[1]);                             \
      if (has_b) {                                                                   \
        pair_hilo<W, 2 * (MT)>(s, kb.x, ah[2], al[2]);                               \
        pair_hilo<W, 2 * (MT) + 1>(s, kb.x, ah[3], al[3]);                           \
      } else {                                                                       \
        ah[2] = ah[3] = al[2] = al[3] = 0u;                                          \
      }                                                                              \
    } else {                                                                         \
      ah[0] = pair_hi<W, 2 * (MT)>(s, ka.x, lane_pair);                              \
      ah[1] = pair_hi<W, 2 * (MT) + 1>(s, ka.x, lane_pair);                          \
      ah[2] = has_b ? pair_hi<W, 2 * (MT)>(s, kb.x, lane_pair) : 0u;                 \
      ah[3] = has_b ? pair_hi<W, 2 * (MT) + 1>(s, kb.x, lane_pair) : 0u;             \
      if constexpr (SPLIT) {                                                         \
        uint32_t dummy;                                                              \
        pair_hilo<W, 2 * (MT)>(s, ka.x, dummy, al[0]);                               \
        pair_hilo<W, 2 * (MT) + 1>(s, ka.x, dummy, al[1]);                           \
        al[2] = al[3] = 0u;                                                          \
        if (has_b) {                                                                 \
          pair_hilo<W, 2 * (MT)>(s, kb.x, dummy, al[2]);                             \
          pair_hilo<W, 2 * (MT) + 1>(s, kb.x, dummy, al[3]);                         \
        }                                                                            \
      }                                                                              \
    }                                                                                \
    mma16816(C[MT], ah, bq.x, bq.y);                                                 \
    if constexpr (SPLIT) {                                                           \
      mma16816(C[MT], ah, bq.z, bq.w);                                               \
      mma16816(C[MT], al, bq.x, bq.y);                                               \
    }                                                                                \
  }
  GTQ_MT(0) GTQ_MT(1) GTQ_MT(2) GTQ_MT(3)
#undef GTQ_MT
}

template <int W, bool SPLIT>
__device__ __forceinline__ void group_scores(const DecodeSmem& s, const uint8_t* tile, int kt0,
                                             int kt1, int koff_lane, uint32_t lane_pair, int lane,
                                             float (&C)[4][4]) {
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int r = 0; r < 4; ++r) C[mt][r] = 0.f;
  for (int kt = kt0; kt < kt1; ++kt)
    ktile_step<W, SPLIT>(s, tile, koff_lane + (kt - kt0) * 128 * W, s.meta.kt_nslots[kt] > 4,
                         lane_pair, s.qf[kt][lane], C);
}

// P.V for one dim tile: V portion of width VB (32 codes, VB words), 4 token k-tiles
template <int VB>
__device__ __forceinline__ void value_tile(const DecodeSmem& s, const uint32_t* pw,
                                           uint32_t lane_pair, const uint32_t (&PB)[4][2],
                                           float (&o)[4]) {
  uint32_t x[VB + 1];
#pragma unroll
  for (int i = 0; i < VB; ++i) x[i] = pw[i];
  x[VB] = 0u;
#define GTQ_V_KTILE(KK)                                                            \
  {                                                                                \
    const uint32_t av[4] = {pair_hi<VB, 4 * (KK)>(s, x, lane_pair),                \
                            pair_hi<VB, 4 * (KK) + 1>(s, x, lane_pair),            \
                            pair_hi<VB, 4 * (KK) + 2>(s, x, lane_pair),            \
                            pair_hi<VB, 4 * (KK) + 3>(s, x, lane_pair)};           \
    mma16816(o, av, PB[KK][0], PB[KK][1]);                                         \
  }
  GTQ_V_KTILE(0) GTQ_V_KTILE(1) GTQ_V_KTILE(2) GTQ_V_KTILE(3)
#undef GTQ_V_KTILE
}

template <int VB>
__global__ void __launch_bounds__(kWarps * 32, 1) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem& s = *reinterpret_cast<DecodeSmem*>(smem_raw);
  const size_t stage_off = (sizeof(DecodeSmem) + 127) & ~size_t(127);
  const int stride = (a.tile_bytes + 127) & ~127;
  const int head = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int nw = blockDim.x >> 5;  // warps in this CTA (<= kWarps)

  if (tid == 0) {
    s.meta = a.meta[head];
    for (int w = 0; w < nw; ++w)
      for (int st = 0; st < kStages; ++st) mbar_init(&s.bar[w][st], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // lookup tables: one 16-byte-vector copy of the prebuilt image
  static_assert(offsetof(DecodeSmem, single) == kPairBytes, "image layout");
  for (int i = tid; i < kDecodeImageBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(s.pair)[i] = a.dec_image[i];
  __syncthreads();
  pdl_launch_dependents();
  const HeadMeta& m = s.meta;
  const int load_bytes = 1024 * (a.kb + VB) + 128 + 128 * m.n_groups;
  const int knorm_off = 1024 * (a.kb + VB) + 128, vnorm_off = 1024 * (a.kb + VB);
  uint32_t lane_pair[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) lane_pair[w] = kPairOff(w) | (uint32_t)(lane * 4);

  // tiles of this split, dealt to warps round-robin; the packed cache does not
  // depend on the previous grid, so its first tiles load before the wait
  const int64_t per = (a.tiles_T + a.splits - 1) / a.splits;
  const int64_t tb0 = (int64_t)split * per, tb1 = min(a.tiles_T, tb0 + per);
  const uint8_t* head_base = a.packed + (size_t)head * a.n_tiles * a.tile_bytes;
  uint8_t* my_stage0 = smem_raw + stage_off + (size_t)(warp * kStages) * stride;
  if (lane == 0) {
    for (int st = 0; st < kStages; ++st) {
      const int64_t tile = tb0 + warp + (int64_t)nw * st;
      if (tile < tb1)
        bulk_load(my_stage0 + (size_t)st * stride, head_base + (size_t)tile * a.tile_bytes,
                  (unsigned)load_bytes, &s.bar[warp][st]);
    }
  }
  // M_h rows of this thread's first rotation task (pos, half of d), prefetched
  // before the wait: they do not depend on the previous grid
  const int rot_pos = tid & (kD - 1), rot_half = (tid >> 7) & 1;
  const bool rot_live = tid < 2 * kD && (rot_pos >> 1) < m.n_slots;
  float4 mv[16];
  if (rot_live) {
    const float4* row = reinterpret_cast<const float4*>(
        a.mrow + ((size_t)head * kD + rot_pos) * kD + 64 * rot_half);
#pragma unroll
    for (int j = 0; j < 16; ++j) mv[j] = row[j];
  }
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
      s.qs[hh][d] = v;
    }
  }
  __syncthreads();
  // q_rot[hh][pos] = M_h[pos] . q[hh] * log2(e) / (sqrt(d) sqrt(m_g)).  Task = (pos,
  // half of d): 16 float4 of the row, 8 query heads; partial sums in s.qf.
  {
    static_assert(sizeof(DecodeSmem::qf) >= 2 * 8 * kD * sizeof(float), "rotation scratch");
    float* part = reinterpret_cast<float*>(s.qf);  // [2][8][128] partial dot products
    for (int task = tid; task < 2 * kD; task += blockDim.x) {
      const int pos = task & (kD - 1), qd = task >> 7;
      const bool live = (pos >> 1) < m.n_slots;
      if (task != tid && live) {  // later tasks of a small CTA: load now
        const float4* row =
            reinterpret_cast<const float4*>(a.mrow + ((size_t)head * kD + pos) * kD + 64 * qd);
#pragma unroll
        for (int j = 0; j < 16; ++j) mv[j] = row[j];
      }
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (live) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int d = 64 * qd + 4 * j;
#pragma unroll
          for (int hh = 0; hh < 8; ++hh) {
            const float4 qv = *reinterpret_cast<const float4*>(&s.qs[hh][d]);
            acc[hh] = fmaf(mv[j].x, qv.x, acc[hh]);
            acc[hh] = fmaf(mv[j].y, qv.y, acc[hh]);
            acc[hh] = fmaf(mv[j].z, qv.z, acc[hh]);
            acc[hh] = fmaf(mv[j].w, qv.w, acc[hh]);
          }
        }
      }
#pragma unroll
      for (int hh = 0; hh < 8; ++hh) part[(qd * 8 + hh) * kD + pos] = acc[hh];
    }
    __syncthreads();
    for (int i = tid; i < 8 * kD; i += blockDim.x) {
      const int hh = i >> 7, pos = i & (kD - 1), slot = pos >> 1;
      // base-2 logits: log2(e) / sqrt(128), and 1/sqrt(m_g) of the group
      const float sc = slot < m.n_slots ? m.inv_sqrt_m[m.slot_group[slot]] *
                                              (1.4426950408889634f * 0.08838834764831845f)
                                        : 0.f;
      s.qr[hh][pos] = (part[(0 * 8 + hh) * kD + pos] + part[(1 * 8 + hh) * kD + pos]) * sc;
    }
  }
  __syncthreads();
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
  bool failed = false;

  int it = 0;
  for (int64_t tile = tb0 + warp; tile < tb1; tile += nw, ++it) {
    const int st = it % kStages;
    const unsigned phase = (unsigned)(it / kStages) & 1u;
    if (!mbar_wait(&s.bar[warp][st], phase)) {
      failed = true;
      break;
    }
    const uint8_t* tl = my_stage0 + (size_t)st * stride;
    const uint32_t* tl32 = reinterpret_cast<const uint32_t*>(tl);

    // ------------------------------------------------------------ scores
    float S[4][4], C[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) S[mt][r] = 0.f;
    for (int gi = 0; gi < m.n_groups; ++gi) {
      const int W = m.grp_width[gi], split = m.grp_split[gi];
      const int kt0 = m.grp_kt0[gi], kt1 = m.grp_kt1[gi];
      const int koff_lane = m.slot_koff[m.grp_first_slot[gi]] + 16 * W * t + 2 * W * g;
      switch (2 * W + split) {
#define GTQ_GROUP(WW)                                                                        \
  case 2 * WW:                                                                               \
    group_scores<WW, false>(s, tl, kt0, kt1, koff_lane, lane_pair[WW < 4 ? WW : 0], lane, C); \
    break;                                                                                   \
  case 2 * WW + 1:                                                                           \
    group_scores<WW, true>(s, tl, kt0, kt1, koff_lane, lane_pair[WW < 4 ? WW : 0], lane, C); \
    break;
        GTQ_GROUP(1) GTQ_GROUP(2) GTQ_GROUP(3) GTQ_GROUP(4)
        GTQ_GROUP(5) GTQ_GROUP(6) GTQ_GROUP(7) GTQ_GROUP(8)
#undef GTQ_GROUP
        default: break;
      }
      // group complete: scale by its fp16 norms
      const uint4 nq = *reinterpret_cast<const uint4*>(tl + knorm_off + gi * 128 + g * 16);
      const __half2* nh = reinterpret_cast<const __half2*>(&nq);
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const float2 n = __half22float2(nh[mt]);
        S[mt][0] = fmaf(n.x, C[mt][0], S[mt][0]);
        S[mt][1] = fmaf(n.x, C[mt][1], S[mt][1]);
        S[mt][2] = fmaf(n.y, C[mt][2], S[mt][2]);
        S[mt][3] = fmaf(n.y, C[mt][3], S[mt][3]);
      }
    }
    // ------------------------------------------------------ online softmax
    const int64_t tok0 = tile * kTile;
    const bool full = tok0 + kTile <= a.T;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = 16 * mt + g + 8 * (r >> 1);
        if (!full && tok0 + j >= a.T) S[mt][r] = -INFINITY;
        mx[r & 1] = fmaxf(mx[r & 1], S[mt][r]);
      }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 4));
      mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 8));
      mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 16));
    }
    float alpha[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const float mn = fmaxf(mrun[hh], mx[hh]);
      alpha[hh] = exp2f(mrun[hh] - mn);
      mrun[hh] = mn;
      lrun[hh] *= alpha[hh];
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
    const uint4 vq = *reinterpret_cast<const uint4*>(tl + vnorm_off + g * 16);
    const __half2* vnh = reinterpret_cast<const __half2*>(&vq);
    uint32_t PB[4][2];
    const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
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
    const uint32_t* vcodes = tl32 + 256 * a.kb;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      value_tile<VB>(s, vcodes + ((i * 8 + g) * 4 + t) * VB, lane_pair[VB < 4 ? VB : 0], PB, O[i]);
    // -------------------------------------------------- refill this stage
    __syncwarp();
    if (lane == 0) {
      const int64_t nxt = tile + (int64_t)nw * kStages;
      if (nxt < tb1) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        bulk_load(my_stage0 + (size_t)st * stride, head_base + (size_t)nxt * a.tile_bytes,
                  (unsigned)load_bytes, &s.bar[warp][st]);
      }
    }
  }
  if (failed && lane == 0) atomicOr(a.status, kStatusTimeout);

  // --------------------------------------------- merge the 4 warps in the CTA
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 4);
    lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 8);
    lrun[hh] += __shfl_xor_sync(0xffffffffu, lrun[hh], 16);
  }
  __syncthreads();  // every warp is done with its stages: reuse them for o
  float* wo = reinterpret_cast<float*>(smem_raw + stage_off);  // [warp][8 heads][128]
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
  float* head_parts = a.partials + (size_t)head * kPartialSlots * 8 * kPartialStride;
  float* part = head_parts + (size_t)split * 8 * kPartialStride;
  for (int idx = tid; idx < 8 * kPartialStride; idx += blockDim.x) {
    const int hh = idx / kPartialStride, k = idx % kPartialStride;
    float v;
    if (k == 0) {
      v = s.hm[hh];
    } else if (k == 1) {
      v = s.hl[hh];
    } else {
      v = 0.f;
      for (int w = 0; w < nw; ++w) v = fmaf(s.wsc[w][hh], wo[(w * 8 + hh) * kD + k - 2], v);
    }
    part[idx] = v;
  }
  // ---------------- merge of the splits.  Every CTA of the head arrives at a
  // per-head barrier (arrival count + generation, bounded spin) once its partial
  // is in global memory; all CTAs of the head are resident (one wave).  Then
  // this CTA merges the outputs it owns: query heads split, split + S, ... when
  // S < G_q; otherwise query head split % G_q and its output dims d with
  // d % nc == split / G_q (nc = CTAs sharing that query head).
  const int S = a.splits, G = a.gq;
  if (S > 1) {
    __syncthreads();
    if (tid == 0) {
      unsigned* bar = a.tickets + (size_t)head * 2;  // [0] arrivals, [1] generation
      const unsigned gen0 = *reinterpret_cast<volatile unsigned*>(&bar[1]);
      __threadfence();
      if (atomicAdd(&bar[0], 1u) == (unsigned)(S - 1)) {
        bar[0] = 0u;
        __threadfence();
        atomicExch(&bar[1], gen0 + 1u);
      } else {
        unsigned spins = 0;
        while (*reinterpret_cast<volatile unsigned*>(&bar[1]) == gen0) {
          if (++spins > kBarrierSpinLimit) {
            atomicOr(a.status, kStatusTimeout);
            break;
          }
          __nanosleep(64);
        }
      }
      __threadfence();
    }
    __syncthreads();
  }
  __syncthreads();  // wo (stage area) fully read before the scratch below reuses it
  float* rot = reinterpret_cast<float*>(smem_raw + stage_off);  // scratch: stages are idle
  const int P = max(1, (int)blockDim.x / kD);                   // threads per output dim
  const int b = head / a.hkv, h = head % a.hkv;
  const int hh0 = S < G ? split : split % G, hh_step = S < G ? S : G;
  const int nc = S < G ? 1 : (S - split % G + G - 1) / G, c = S < G ? 0 : split / G;
  for (int hh = hh0; hh < G; hh += hh_step) {
    // merged o_rot[hh][:]: P threads per dim, each over splits j = p, p + P, ...
    for (int idx = tid; idx < P * kD; idx += blockDim.x) {
      const int p = idx / kD, d = idx % kD;
      const float* q = head_parts + hh * kPartialStride;
      float M = -1e30f, L = 0.f, o = 0.f;
      for (int j0 = p; j0 < S; j0 += 16 * P) {
        float vm[16], vl[16], vo[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int j = j0 + k * P;
          const bool in = j < S;
          const float* pj = q + (size_t)j * 8 * kPartialStride;
          vm[k] = in ? __ldcg(pj) : -1e30f;
          vl[k] = in ? __ldcg(pj + 1) : 0.f;
          vo[k] = in ? __ldcg(pj + 2 + d) : 0.f;
        }
        float mc = vm[0];
#pragma unroll
        for (int k = 1; k < 16; ++k) mc = fmaxf(mc, vm[k]);
        const float mn = fmaxf(M, mc), sc = exp2f(M - mn);
        L *= sc;
        o *= sc;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float w = exp2f(vm[k] - mn);
          L = fmaf(w, vl[k], L);
          o = fmaf(w, vo[k], o);
        }
        M = mn;
      }
      rot[(p * 3 + 0) * kD + d] = M;
      rot[(p * 3 + 1) * kD + d] = L;
      rot[(p * 3 + 2) * kD + d] = o;
    }
    __syncthreads();
    for (int d = tid; d < kD; d += blockDim.x) {
      float M = -1e30f;
      for (int p = 0; p < P; ++p) M = fmaxf(M, rot[(p * 3) * kD + d]);
      float L = 0.f, o = 0.f;
      for (int p = 0; p < P; ++p) {
        const float w = exp2f(rot[(p * 3) * kD + d] - M);
        L = fmaf(w, rot[(p * 3 + 1) * kD + d], L);
        o = fmaf(w, rot[(p * 3 + 2) * kD + d], o);
      }
      s.qs[0][d] = o / L;  // o_rot[hh][d]
    }
    __syncthreads();
    // out[dd] = sum_r R_V[r][dd] o_rot[r] for this CTA's dims dd = c, c + nc, ...:
    // 16 lanes per dim, 8 rows each
    const int n_dims = (kD - c + nc - 1) / nc;
    const int n_items = ((n_dims * 16 + 31) / 32) * 32;  // whole warps: the shuffles need every lane
    for (int idx = tid; idx < n_items; idx += blockDim.x) {
      const bool valid = idx < n_dims * 16;
      const int dd = c + (idx >> 4) * nc, r0 = (idx & 15) * 8;
      float acc = 0.f;
      if (valid) {
#pragma unroll
        for (int r = r0; r < r0 + 8; ++r) acc = fmaf(__ldg(a.rot_v + r * kD + dd), s.qs[0][r], acc);
      }
#pragma unroll
      for (int o = 8; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, 16);
      if (valid && (idx & 15) == 0)
        a.out[((size_t)b * a.hkv * a.gq + (size_t)h * a.gq + hh) * kD + dd] = acc;
    }
    __syncthreads();
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
  a.mrow = p->d_mrow;
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
  int nw = (int)std::min<size_t>(kWarps, (dev_smem - stage_off) / (stride * kStages));
  nw = std::max(nw, 1);
  // stages; reused at the end for the warps' o (nw x 4 KB) and R_V (128 x 129 floats)
  const size_t smem = stage_off + std::max({stride * nw * kStages, (size_t)nw * 8 * kD * 4,
                                            (size_t)kD * (kD + 1) * 4});
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
  splits = (int)std::min<int64_t>(splits, (a.tiles_T + nw - 1) / nw);
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
