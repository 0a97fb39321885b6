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
#include <cmath>

#include "gtq_internal.h"

namespace gtq {
namespace {

constexpr int kWarps = 12;  // one CTA per SM: up to 12 warps, 2 private tile stages each
constexpr int kStages = 2;
constexpr unsigned kSpinLimit = 1u << 26;

struct DecodeArgs {
  const uint8_t* packed;
  const HeadMeta* meta;
  const float* qrot;  // [heads][8][128]
  const __half* lut_hi;
  const __half* lut_lo;
  float* partials;    // [heads][kMaxSplits][8][kPartialStride]
  int* status;
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

// d = a.b (accumulator starts at zero)
__device__ inline void mma16816_zero(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                     uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ inline uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
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
// Single-code tables (fp16 hi and lo parts, widths 1..8, 2^w entries): at byte
// offset 1024 - 2^(w+2) inside a 1 KB region, so offset | code * 2 needs no add;
// widths up to 6 occupy at most 32 banks and never conflict.
// ---------------------------------------------------------------------------
constexpr int kPairBytes = 10752;
__host__ __device__ constexpr uint32_t kPairOff(int w) { return w == 3 ? 0u : (w == 2 ? 8192u : 10240u); }
__host__ __device__ constexpr uint32_t kSingleOff(int w) { return 1024u - (4u << w); }

struct DecodeSmem {
  uint32_t pair[kPairBytes / 4];
  __half single_hi[512];
  __half single_lo[512];
  uint4 qf[kMaxKt][32];  // per k-tile & lane: hi(slot A), hi(slot B), lo(A), lo(B)
  HeadMeta meta;
  uint64_t bar[kWarps][kStages];
  float wm[kWarps][8], wl[kWarps][8];
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
__device__ __forceinline__ uint16_t lds16_hi(const DecodeSmem& s, uint32_t byte_off) {
  return *reinterpret_cast<const uint16_t*>(reinterpret_cast<const uint8_t*>(s.single_hi) + byte_off);
}
__device__ __forceinline__ uint16_t lds16_lo(const DecodeSmem& s, uint32_t byte_off) {
  return *reinterpret_cast<const uint16_t*>(reinterpret_cast<const uint8_t*>(s.single_lo) + byte_off);
}

// half2 of codes (2x, 2x+1), width W, from the bit string x (pair at bits [2xW, 2xW + 2W))
template <int W, int X>
__device__ __forceinline__ uint32_t pair_hi(const DecodeSmem& s, const uint32_t* x, uint32_t lane_pair) {
  if constexpr (W <= 3) {
    return lds32(s, fld<2 * X * W, 2 * W, 7>(x, lane_pair));
  } else {
    const uint32_t a0 = fld<2 * X * W, W, 1>(x, kSingleOff(W));
    const uint32_t a1 = fld<(2 * X + 1) * W, W, 1>(x, kSingleOff(W));
    return (uint32_t)lds16_hi(s, a0) | ((uint32_t)lds16_hi(s, a1) << 16);
  }
}
template <int W, int X>
__device__ __forceinline__ uint32_t pair_lo(const DecodeSmem& s, const uint32_t* x) {
  const uint32_t a0 = fld<2 * X * W, W, 1>(x, kSingleOff(W));
  const uint32_t a1 = fld<(2 * X + 1) * W, W, 1>(x, kSingleOff(W));
  return (uint32_t)lds16_lo(s, a0) | ((uint32_t)lds16_lo(s, a1) << 16);
}

// The 16w-bit portion of one key slot for this lane (tokens g + 8u, u = 0..7),
// realigned to bit 0 of x[] (portions start at an even byte).
template <int W>
struct KeyWords {
  static constexpr int NW = (16 * W + 31) / 32 + 1;
  uint32_t x[NW];
  __device__ __forceinline__ void load(const uint8_t* tile, int byte_off) {
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(tile + (byte_off & ~3));
#pragma unroll
    for (int i = 0; i < NW; ++i) x[i] = wp[i];
    if (byte_off & 2) {
#pragma unroll
      for (int i = 0; i + 1 < NW; ++i) x[i] = __funnelshift_r(x[i], x[i + 1], 16);
    }
  }
};

// A fragments (rows: tokens; cols: the k-tile's 16 coords) of a group-pure k-tile:
// slot A (first + t) feeds regs 0/1, slot B (first + t + 4) regs 2/3.
#define GTQ_A_HI(KA, KB, U) \
  { a[(U) >> 1][(U)&1] = pair_hi<W, U>(s, KA.x, lane_pair); \
    a[(U) >> 1][2 + ((U)&1)] = has_b ? pair_hi<W, U>(s, KB.x, lane_pair) : 0u; }
#define GTQ_A_LO(KA, KB, U) \
  { a[(U) >> 1][(U)&1] = pair_lo<W, U>(s, KA.x); \
    a[(U) >> 1][2 + ((U)&1)] = has_b ? pair_lo<W, U>(s, KB.x) : 0u; }

template <int W>
__device__ __forceinline__ void key_ktile(const DecodeSmem& s, const uint8_t* tile, int koff_a,
                                          bool has_b, uint32_t lane_pair, bool split, bool first,
                                          const uint4& bq, float (&C)[4][4], float (&Cc)[4][4]) {
  KeyWords<W> ka, kb;
  ka.load(tile, koff_a);
  if (has_b) kb.load(tile, koff_a + 64 * W);
  uint32_t a[4][4];
  GTQ_A_HI(ka, kb, 0) GTQ_A_HI(ka, kb, 1) GTQ_A_HI(ka, kb, 2) GTQ_A_HI(ka, kb, 3)
  GTQ_A_HI(ka, kb, 4) GTQ_A_HI(ka, kb, 5) GTQ_A_HI(ka, kb, 6) GTQ_A_HI(ka, kb, 7)
  if (first) {
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) mma16816_zero(C[mt], a[mt], bq.x, bq.y);
  } else {
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) mma16816(C[mt], a[mt], bq.x, bq.y);
  }
  if (split) {  // hi.lo + lo.hi correction terms of the split fp16 product
    if (first) {
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) mma16816_zero(Cc[mt], a[mt], bq.z, bq.w);
    } else {
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) mma16816(Cc[mt], a[mt], bq.z, bq.w);
    }
    GTQ_A_LO(ka, kb, 0) GTQ_A_LO(ka, kb, 1) GTQ_A_LO(ka, kb, 2) GTQ_A_LO(ka, kb, 3)
    GTQ_A_LO(ka, kb, 4) GTQ_A_LO(ka, kb, 5) GTQ_A_LO(ka, kb, 6) GTQ_A_LO(ka, kb, 7)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) mma16816(Cc[mt], a[mt], bq.x, bq.y);
  }
}
#undef GTQ_A_HI
#undef GTQ_A_LO

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
  // lookup tables
  for (int i = tid; i < (4 + 16 + 64) * 32; i += blockDim.x) {
    const int ln = i & 31, e = i >> 5;
    const int w = e < 4 ? 1 : (e < 20 ? 2 : 3);
    const int idx = e - (w == 1 ? 0 : (w == 2 ? 4 : 20));
    const int c0 = idx & ((1 << w) - 1), c1 = idx >> w;
    s.pair[(kPairOff(w) >> 2) + idx * 32 + ln] =
        pack_half2(a.lut_hi[lut_base(w) + c0], a.lut_hi[lut_base(w) + c1]);
  }
  for (int i = tid; i < kLutEntries; i += blockDim.x) {
    int w = 1;
    while (i >= lut_base(w + 1)) ++w;
    const int c = i - lut_base(w);
    s.single_hi[(kSingleOff(w) >> 1) + c] = a.lut_hi[i];
    s.single_lo[(kSingleOff(w) >> 1) + c] = a.lut_lo[i];
  }
  __syncthreads();
  const HeadMeta& m = s.meta;
  const int load_bytes = 1024 * (a.kb + VB) + 128 + 128 * m.n_groups;
  const int knorm_off = 1024 * (a.kb + VB) + 128, vnorm_off = 1024 * (a.kb + VB);
  uint32_t lane_pair[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) lane_pair[w] = kPairOff(w) | (uint32_t)(lane * 4);
  // B fragments (query) of every decode k-tile; slots past the k-tile's run are zero
  {
    const float* qh = a.qrot + (size_t)head * 8 * kD;
    for (int idx = tid; idx < m.n_ktiles * 32; idx += blockDim.x) {
      const int kt = idx >> 5, ln = idx & 31, gg = ln >> 2, tt = ln & 3;
      uint32_t out[4];
      for (int half = 0; half < 2; ++half) {
        const int sl = tt + 4 * half;  // slot within the k-tile
        const bool in = sl < m.kt_nslots[kt];
        const int pos = 2 * (m.kt_first_slot[kt] + sl);
        const float v0 = in ? qh[gg * kD + pos] : 0.f, v1 = in ? qh[gg * kD + pos + 1] : 0.f;
        const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
        out[half] = pack_half2(h0, h1);
        out[2 + half] = pack_half2(__float2half_rn(v0 - __half2float(h0)),
                                   __float2half_rn(v1 - __half2float(h1)));
      }
      s.qf[kt][ln] = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
  __syncthreads();

  // tiles of this split, dealt to warps round-robin
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
  __syncwarp();

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
    float S[4][4], C[4][4], Cc[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) S[mt][r] = C[mt][r] = Cc[mt][r] = 0.f;
    for (int kt = 0; kt < m.n_ktiles; ++kt) {
      const int grp = m.kt_group[kt], W = m.grp_width[grp], flags = m.kt_flags[kt];
      const bool split = m.grp_split[grp], first = flags & 1, has_b = m.kt_nslots[kt] > 4;
      const int koff_a = m.slot_koff[m.kt_first_slot[kt]] + 16 * W * t + 2 * W * g;
      const uint4 bq = s.qf[kt][lane];
      switch (W) {
        case 1: key_ktile<1>(s, tl, koff_a, has_b, lane_pair[1], split, first, bq, C, Cc); break;
        case 2: key_ktile<2>(s, tl, koff_a, has_b, lane_pair[2], split, first, bq, C, Cc); break;
        case 3: key_ktile<3>(s, tl, koff_a, has_b, lane_pair[3], split, first, bq, C, Cc); break;
        case 4: key_ktile<4>(s, tl, koff_a, has_b, 0u, split, first, bq, C, Cc); break;
        case 5: key_ktile<5>(s, tl, koff_a, has_b, 0u, split, first, bq, C, Cc); break;
        case 6: key_ktile<6>(s, tl, koff_a, has_b, 0u, split, first, bq, C, Cc); break;
        case 7: key_ktile<7>(s, tl, koff_a, has_b, 0u, split, first, bq, C, Cc); break;
        default: key_ktile<8>(s, tl, koff_a, has_b, 0u, split, first, bq, C, Cc); break;
      }
      if (flags & 2) {  // group complete: scale by its fp16 norms
        const uint4 nq = *reinterpret_cast<const uint4*>(tl + knorm_off + grp * 128 + g * 16);
        const __half2* nh = reinterpret_cast<const __half2*>(&nq);
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const float2 n = __half22float2(nh[mt]);
          if (split) {
#pragma unroll
            for (int r = 0; r < 4; ++r) C[mt][r] += Cc[mt][r];
          }
          S[mt][0] = fmaf(n.x, C[mt][0], S[mt][0]);
          S[mt][1] = fmaf(n.x, C[mt][1], S[mt][1]);
          S[mt][2] = fmaf(n.y, C[mt][2], S[mt][2]);
          S[mt][3] = fmaf(n.y, C[mt][3], S[mt][3]);
        }
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
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      O[i][0] *= alpha[0];
      O[i][2] *= alpha[0];
      O[i][1] *= alpha[1];
      O[i][3] *= alpha[1];
    }
    const uint4 vq = *reinterpret_cast<const uint4*>(tl + vnorm_off + g * 16);
    const __half2* vnh = reinterpret_cast<const __half2*>(&vq);
    uint32_t PB[4][2];
    const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const float2 vn = __half22float2(vnh[mt]);
      float pp[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = 16 * mt + g + 8 * (r >> 1);
        const float p = exp2f(S[mt][r] - mrun[r & 1]);
        lrun[r & 1] += p;
        const float nv = (r >> 1) ? vn.y : vn.x;
        pp[r] = (full || tok0 + j < a.T) ? p * nv * inv_sqrt_d : 0.f;
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
  float* part = a.partials + ((size_t)head * kMaxSplits + split) * 8 * kPartialStride;
  for (int idx = tid; idx < 8 * kPartialStride; idx += blockDim.x) {
    const int hh = idx / kPartialStride, k = idx % kPartialStride;
    float M = -1e30f;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, s.wm[w][hh]);
    float v = 0.f;
    for (int w = 0; w < nw; ++w) {
      const float sc = exp2f(s.wm[w][hh] - M);
      v += sc * (k == 1 ? s.wl[w][hh] : (k >= 2 ? wo[(w * 8 + hh) * kD + k - 2] : 0.f));
    }
    part[idx] = k == 0 ? M : v;
  }
}

// grid (heads * g_q); 128 threads; q [B][Hq][128]
template <typename T>
__global__ void __launch_bounds__(128) rotate_q_kernel(const T* __restrict__ q,
                                                       const HeadMeta* __restrict__ meta,
                                                       const float* __restrict__ mrow, int hkv,
                                                       int g_q, float* __restrict__ qrot) {
  const int head = blockIdx.x / 8, hh = blockIdx.x % 8;
  const int b = head / hkv, h = head % hkv;
  const int pos = threadIdx.x;
  __shared__ float qs[kD];
  const bool live = hh < g_q;
  qs[pos] = live ? (float)q[((size_t)b * hkv * g_q + (size_t)h * g_q + hh) * kD + pos] : 0.f;
  __syncthreads();
  const HeadMeta& m = meta[head];
  const int slot = pos >> 1;
  float v = 0.f;
  if (live && slot < m.n_slots) {
    const float* row = mrow + ((size_t)head * kD + pos) * kD;
    for (int d = 0; d < kD; ++d) v = fmaf(row[d], qs[d], v);
    // log2(e) / sqrt(128): scores come out in base-2 logits
    v *= m.inv_sqrt_m[m.slot_group[slot]] * (1.4426950408889634f * 0.08838834764831845f);
  }
  qrot[((size_t)head * 8 + hh) * kD + pos] = v;
}

// grid (heads, g_q); 128 threads
__global__ void __launch_bounds__(128) merge_kernel(const float* __restrict__ partials, int splits,
                                                    const float* __restrict__ rot_v, int hkv,
                                                    int g_q, float* __restrict__ out) {
  const int head = blockIdx.x, hh = blockIdx.y, tid = threadIdx.x;
  const int b = head / hkv, h = head % hkv;
  __shared__ float wsc[kMaxSplits];
  __shared__ float red[128];
  __shared__ float orot[kD];
  const float* P = partials + (size_t)head * kMaxSplits * 8 * kPartialStride + hh * kPartialStride;
  const size_t sstride = 8 * kPartialStride;
  float M = -1e30f;
  for (int sp = tid; sp < splits; sp += 128) M = fmaxf(M, P[sp * sstride]);
  red[tid] = M;
  __syncthreads();
  for (int off = 64; off; off >>= 1) {
    if (tid < off) red[tid] = fmaxf(red[tid], red[tid + off]);
    __syncthreads();
  }
  M = red[0];
  __syncthreads();
  float L = 0.f;
  for (int sp = tid; sp < splits; sp += 128) {
    const float w = exp2f(P[sp * sstride] - M);
    wsc[sp] = w;
    L += w * P[sp * sstride + 1];
  }
  red[tid] = L;
  __syncthreads();
  for (int off = 64; off; off >>= 1) {
    if (tid < off) red[tid] += red[tid + off];
    __syncthreads();
  }
  L = red[0];
  float o = 0.f;
  for (int sp = 0; sp < splits; ++sp) o = fmaf(wsc[sp], P[sp * sstride + 2 + tid], o);
  orot[tid] = o / L;
  __syncthreads();
  float r = 0.f;
  for (int k = 0; k < kD; ++k) r = fmaf(rot_v[k * kD + tid], orot[k], r);  // (R_V^T o_rot)[tid]
  out[((size_t)b * hkv * g_q + (size_t)h * g_q + hh) * kD + tid] = r;
}

}  // namespace

cudaError_t launch_decode(const gtq_plan* p, const uint8_t* packed, int64_t T, const void* q,
                          int q_dtype, float* out, cudaStream_t s) {
  const int hkv = p->cfg.n_kv_heads, gq = p->g_q;
  if (q_dtype == GTQ_DTYPE_FP16)
    rotate_q_kernel<__half><<<p->n_heads * 8, 128, 0, s>>>((const __half*)q, p->d_meta,
                                                           p->d_mrow, hkv, gq, p->d_qrot);
  else
    rotate_q_kernel<float><<<p->n_heads * 8, 128, 0, s>>>((const float*)q, p->d_meta, p->d_mrow,
                                                          hkv, gq, p->d_qrot);
  DecodeArgs a;
  a.packed = packed;
  a.meta = p->d_meta;
  a.qrot = p->d_qrot;
  a.lut_hi = p->tab.lut_hi;
  a.lut_lo = p->tab.lut_lo;
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
  const size_t smem = stage_off + std::max(stride * nw * kStages, (size_t)nw * 8 * kD * 4);
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
  const int target = std::max(1, per_sm) * p->n_sms;
  int splits = (target + p->n_heads - 1) / p->n_heads;
  splits = (int)std::min<int64_t>(splits, (a.tiles_T + nw - 1) / nw);
  splits = std::max(1, std::min(splits, kMaxSplits));
  // every split must own at least one tile
  const int64_t per = (a.tiles_T + splits - 1) / splits;
  splits = (int)((a.tiles_T + per - 1) / per);
  a.splits = splits;
  cudaError_t e = cudaErrorInvalidValue;
  switch (a.vb) {
#define GTQ_LAUNCH_VB(VB)                                                                       \
  case VB:                                                                                     \
    e = cudaFuncSetAttribute(decode_kernel<VB>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                             (int)smem);                                                        \
    if (e == cudaSuccess) decode_kernel<VB><<<dim3(splits, p->n_heads), nw * 32, smem, s>>>(a); \
    break;
    GTQ_LAUNCH_VB(1) GTQ_LAUNCH_VB(2) GTQ_LAUNCH_VB(3) GTQ_LAUNCH_VB(4)
    GTQ_LAUNCH_VB(5) GTQ_LAUNCH_VB(6) GTQ_LAUNCH_VB(7) GTQ_LAUNCH_VB(8)
#undef GTQ_LAUNCH_VB
  }
  if (e != cudaSuccess) return e;
  merge_kernel<<<dim3(p->n_heads, gq), 128, 0, s>>>(p->d_partials, splits, p->tab.rot_v, hkv,
                                                    gq, out);
  return cudaGetLastError();
}

}  // namespace gtq
