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

constexpr int kWarps = 4;
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
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ inline uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ inline uint32_t pack_half2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// w-bit code at bit offset `bit` of a 4-byte-aligned word array in shared memory
__device__ inline uint32_t get_bits(const uint32_t* words, int bit, int w) {
  const int wd = bit >> 5, sh = bit & 31;
  const uint64_t v = ((uint64_t)words[wd + 1] << 32) | words[wd];
  return (uint32_t)(v >> sh) & ((1u << w) - 1);
}

struct DecodeSmem {
  uint4 qf[kMaxSegs][32];  // per segment & lane: hi(slot A), hi(slot B), lo(A), lo(B)
  __half lut_hi[kLutEntries + 2];
  __half lut_lo[kLutEntries + 2];
  HeadMeta meta;
  uint64_t bar[kWarps][kStages];
  float wm[kWarps][8], wl[kWarps][8];
};

// A fragments of one key slot for the 4 m-tiles: regs[mt][r0], regs[mt][r0 + 1]
__device__ inline void key_slot_frags(const DecodeSmem& s, const uint32_t* tile32, int slot, int g,
                                      bool want_lo, uint32_t (&hi)[4][4], uint32_t (&lo)[4][4],
                                      int r0) {
  const HeadMeta& m = s.meta;
  const int w = slot < m.n_slots ? m.slot_width[slot] : 0;
  if (w == 0) {
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      hi[mt][r0] = hi[mt][r0 + 1] = 0u;
      lo[mt][r0] = lo[mt][r0 + 1] = 0u;
    }
    return;
  }
  const uint32_t* base = tile32 + m.slot_koff[slot] / 4;
  const int lb = lut_base(w);
  const bool split = want_lo && m.grp_split[m.slot_group[slot]];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int bit = g * 16 * w + 2 * u * w;
    const uint32_t c0 = get_bits(base, bit, w), c1 = get_bits(base, bit + w, w);
    const uint32_t vh = pack_half2(s.lut_hi[lb + c0], s.lut_hi[lb + c1]);
    const uint32_t vl = split ? pack_half2(s.lut_lo[lb + c0], s.lut_lo[lb + c1]) : 0u;
    hi[u >> 1][r0 + (u & 1)] = vh;
    lo[u >> 1][r0 + (u & 1)] = vl;
  }
}

__global__ void __launch_bounds__(kWarps * 32) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem& s = *reinterpret_cast<DecodeSmem*>(smem_raw);
  const size_t stage_off = (sizeof(DecodeSmem) + 127) & ~size_t(127);
  const int stride = (a.tile_bytes + 127) & ~127;
  const int head = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;

  if (tid == 0) {
    s.meta = a.meta[head];
    for (int w = 0; w < kWarps; ++w)
      for (int st = 0; st < kStages; ++st) mbar_init(&s.bar[w][st], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < kLutEntries; i += blockDim.x) {
    s.lut_hi[i] = a.lut_hi[i];
    s.lut_lo[i] = a.lut_lo[i];
  }
  __syncthreads();
  const HeadMeta& m = s.meta;
  const int load_bytes = 1024 * (a.kb + a.vb) + 128 + 128 * m.n_groups;
  const int knorm_off = 1024 * (a.kb + a.vb) + 128, vnorm_off = 1024 * (a.kb + a.vb);
  // B fragments (query), masked per segment
  {
    const float* qh = a.qrot + (size_t)head * 8 * kD;
    for (int idx = tid; idx < m.n_segs * 32; idx += blockDim.x) {
      const int sg = idx >> 5, ln = idx & 31, gg = ln >> 2, tt = ln & 3;
      int kt = 0;
      while (kt < 7 && !(sg >= m.kt_seg_start[kt] && sg < m.kt_seg_start[kt] + m.kt_seg_count[kt]))
        ++kt;
      uint32_t out[4];
      for (int half = 0; half < 2; ++half) {
        const int sl = tt + 4 * half;  // slot within the k-tile
        const bool in = sl >= m.seg_lo[sg] && sl < m.seg_hi[sg];
        const int pos = 2 * (8 * kt + sl);
        const float v0 = in ? qh[gg * kD + pos] : 0.f, v1 = in ? qh[gg * kD + pos + 1] : 0.f;
        const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
        out[half] = pack_half2(h0, h1);
        out[2 + half] = pack_half2(__float2half_rn(v0 - __half2float(h0)),
                                   __float2half_rn(v1 - __half2float(h1)));
      }
      s.qf[sg][ln] = make_uint4(out[0], out[1], out[2], out[3]);
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
      const int64_t tile = tb0 + warp + (int64_t)kWarps * st;
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
  for (int64_t tile = tb0 + warp; tile < tb1; tile += kWarps, ++it) {
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
      for (int r = 0; r < 4; ++r) S[mt][r] = C[mt][r] = 0.f;
    for (int kt = 0; kt < m.n_ktiles; ++kt) {
      uint32_t Ah[4][4], Al[4][4];
      key_slot_frags(s, tl32, 8 * kt + t, g, true, Ah, Al, 0);
      key_slot_frags(s, tl32, 8 * kt + t + 4, g, true, Ah, Al, 2);
      const int sg0 = m.kt_seg_start[kt], sg1 = sg0 + m.kt_seg_count[kt];
      for (int sg = sg0; sg < sg1; ++sg) {
        const uint4 bq = s.qf[sg][lane];
        const int grp = m.seg_group[sg];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) mma16816(C[mt], Ah[mt], bq.x, bq.y);
        if (m.grp_split[grp]) {
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
            mma16816(C[mt], Ah[mt], bq.z, bq.w);
            mma16816(C[mt], Al[mt], bq.x, bq.y);
          }
        }
        if (m.seg_last[sg]) {
          const __half* kn = reinterpret_cast<const __half*>(tl + knorm_off + grp * 128 + g * 16);
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
            const float n0 = __half2float(kn[2 * mt]), n1 = __half2float(kn[2 * mt + 1]);
            S[mt][0] = fmaf(n0, C[mt][0], S[mt][0]);
            S[mt][1] = fmaf(n0, C[mt][1], S[mt][1]);
            S[mt][2] = fmaf(n1, C[mt][2], S[mt][2]);
            S[mt][3] = fmaf(n1, C[mt][3], S[mt][3]);
            C[mt][0] = C[mt][1] = C[mt][2] = C[mt][3] = 0.f;
          }
        }
      }
    }
    // ------------------------------------------------------ online softmax
    const int64_t tok0 = tile * kTile;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = 16 * mt + g + 8 * (r >> 1);
        if (tok0 + j >= a.T) S[mt][r] = -INFINITY;
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
    const __half* vn = reinterpret_cast<const __half*>(tl + vnorm_off + g * 16);
    uint32_t PB[4][2];
    const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      float pp[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = 16 * mt + g + 8 * (r >> 1);
        const float p = exp2f(S[mt][r] - mrun[r & 1]);
        lrun[r & 1] += p;
        pp[r] = (tok0 + j < a.T) ? p * __half2float(vn[2 * mt + (r >> 1)]) * inv_sqrt_d : 0.f;
      }
      const uint32_t x0 = pack_half2(__float2half_rn(pp[0]), __float2half_rn(pp[1]));
      const uint32_t x1 = pack_half2(__float2half_rn(pp[2]), __float2half_rn(pp[3]));
      PB[mt][0] = movmatrix_t(x0);
      PB[mt][1] = movmatrix_t(x1);
    }
    // ---------------------------------------------------------------- P.V
    const uint32_t* vcodes = tl32 + (1024 * a.kb) / 4;
    const int vlb = lut_base(a.vb);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t* pw = vcodes + ((i * 8 + g) * 4 + t) * a.vb;
      uint32_t Av[4][4];
#pragma unroll
      for (int x2 = 0; x2 < 16; ++x2) {
        const uint32_t c0 = get_bits(pw, 2 * x2 * a.vb, a.vb);
        const uint32_t c1 = get_bits(pw, (2 * x2 + 1) * a.vb, a.vb);
        Av[x2 >> 2][x2 & 3] = pack_half2(s.lut_hi[vlb + c0], s.lut_hi[vlb + c1]);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) mma16816(O[i], Av[kk], PB[kk][0], PB[kk][1]);
    }
    // -------------------------------------------------- refill this stage
    __syncwarp();
    if (lane == 0) {
      const int64_t nxt = tile + (int64_t)kWarps * kStages;
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
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s.wm[w][hh]);
    float v = 0.f;
    for (int w = 0; w < kWarps; ++w) {
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
  const int target = 2 * p->n_sms;
  int splits = (target + p->n_heads - 1) / p->n_heads;
  splits = (int)std::min<int64_t>(splits, (a.tiles_T + kWarps - 1) / kWarps);
  splits = std::max(1, std::min(splits, kMaxSplits));
  // every split must own at least one tile
  const int64_t per = (a.tiles_T + splits - 1) / splits;
  splits = (int)((a.tiles_T + per - 1) / per);
  a.splits = splits;
  const size_t stage_off = (sizeof(DecodeSmem) + 127) & ~size_t(127);
  const size_t stride = (p->tile_bytes + 127) & ~size_t(127);
  size_t smem = stage_off + std::max(stride * kWarps * kStages, (size_t)kWarps * 8 * kD * 4);
  cudaError_t e =
      cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_kernel<<<dim3(splits, p->n_heads), kWarps * 32, smem, s>>>(a);
  merge_kernel<<<dim3(p->n_heads, gq), 128, 0, s>>>(p->d_partials, splits, p->tab.rot_v, hkv,
                                                    gq, out);
  return cudaGetLastError();
}

}  // namespace gtq
