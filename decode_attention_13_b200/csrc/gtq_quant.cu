// TurboQuant-MSE quantize-pack of keys (Block-GTQ mixed widths) and values
// (uniform width) into the packed cache ("RoPE-Aware Bit Allocation for
// KV-Cache Quantization", Abstract: Block-GTQ uses TurboQuant-MSE as its base
// quantizer, and the page serves decoding from the packed codes).
//
// Per token and key group g (width w, m coordinates): n = ||k_g|| (fp64 sum of
// exact squares, blocks ascending, p0 then p1), y = (sqrt(m)/n) (M_h k)[rows of
// g] with M_h the block-diagonal rotation in packed order, code = number of
// fp32 thresholds below the fp32 value y; n = 0 gives codes 0.  Values: one
// group of the 128 dims with R_V.  Stored norm: fp16(n), round-to-nearest-even
// from fp64, clamped to 65504 (clamping raises GTQ_ERR_OVERFLOW in the status).
//
// This kernel computes the rotation on CUDA cores in fp32: one CTA walks
// 64-token tiles of one head with M_h and R_V resident in shared memory, builds
// the packed tile image in shared memory and writes it with 16-byte stores.
#include <cmath>

#include "gtq_internal.h"

namespace gtq {
namespace {

constexpr int kQThreads = 256;

struct QuantArgs {
  const void* k;
  const void* v;
  int64_t s0, s1, s2;
  int64_t t0, n;
  uint8_t* packed;
  const HeadMeta* meta;
  const float* mrow;
  const float* rot_v;
  const float* thr;
  int hkv;
  int pairing;
  int64_t n_tiles;
  int tile_bytes;
  int kb, vb;
  int* status;
  SeqMap sm;       // tile addresses and sequence lengths
  int64_t cap;     // t_capacity: lengths are clamped to it
};

struct QuantSmem {
  float mt[kD][kD];      // M_h^T: mt[dim][pos]
  float rt[kD][kD];      // R_V^T: rt[dim][row]
  float x[kD][kTile];    // current K or V tile, dim-major
  uint8_t codes[kTile][kD];
  float scale[kTile][kMaxGroups];
  float thr[kThrEntries];
  HeadMeta meta;
  int overflow;
};

// the tile image follows QuantSmem, rounded up so that 16-byte accesses are aligned
constexpr size_t kImgOffset = (sizeof(QuantSmem) + 127) & ~size_t(127);

__device__ inline int lm_code(float y, const float* thr, int w) {
  const float* t = thr + thr_base(w);
  int lo = 0;
  for (int step = 1 << (w - 1); step; step >>= 1)
    if (y > t[lo + step - 1]) lo += step;
  return lo;
}

// write `code` (w bits) at bit offset `bit` of a 32-bit-word array (clear, then set)
__device__ inline void put_bits(uint32_t* words, int bit, uint32_t code, int w) {
  const int wd = bit >> 5, sh = bit & 31;
  const uint64_t mask = ((1ull << w) - 1) << sh;
  const uint64_t val = ((uint64_t)code << sh) & mask;
  words[wd] = (words[wd] & ~(uint32_t)mask) | (uint32_t)val;
  if (sh + w > 32)
    words[wd + 1] = (words[wd + 1] & ~(uint32_t)(mask >> 32)) | (uint32_t)(val >> 32);
}

template <typename T>
__device__ inline float ld_elem(const T* p);
template <>
__device__ inline float ld_elem<__half>(const __half* p) { return __half2float(*p); }
template <>
__device__ inline float ld_elem<float>(const float* p) { return *p; }

__device__ inline __half norm_to_half(double n, int* overflow) {
  if (n > 65504.0) {
    *overflow = 1;
    n = 65504.0;
  }
  return __double2half(n);  // round-to-nearest-even from fp64
}

template <typename T>
__device__ void load_tile(QuantSmem& s, const T* base, int64_t tok0, int64_t t0, int64_t n,
                          int64_t s2) {
  for (int idx = threadIdx.x; idx < kTile * kD; idx += kQThreads) {
    const int j = idx / kD, d = idx % kD;
    const int64_t t = tok0 + j;
    s.x[d][j] = (t >= t0 && t < t0 + n) ? ld_elem<T>(base + t * s2 + d) : 0.f;
  }
}

// y[4 tokens][8 rows] = x^T rot^T for this thread's (token block tb, row block rb)
__device__ inline void small_gemm(const float (*rot)[kD], const float (*x)[kTile], int tb, int rb,
                                  float (&y)[4][8]) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) y[a][c] = 0.f;
#pragma unroll 4
  for (int d = 0; d < kD; ++d) {
    const float4 xv = *reinterpret_cast<const float4*>(&x[d][4 * tb]);
    const float4 r0 = *reinterpret_cast<const float4*>(&rot[d][8 * rb]);
    const float4 r1 = *reinterpret_cast<const float4*>(&rot[d][8 * rb + 4]);
    const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
    const float rs[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
    for (int a2 = 0; a2 < 4; ++a2)
#pragma unroll
      for (int c = 0; c < 8; ++c) y[a2][c] = fmaf(xs[a2], rs[c], y[a2][c]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kQThreads, 1) quantize_kernel(QuantArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  QuantSmem& s = *reinterpret_cast<QuantSmem*>(smem_raw);
  uint8_t* img = smem_raw + kImgOffset;  // tile image, a.tile_bytes (16-byte accesses)
  uint32_t* img32 = reinterpret_cast<uint32_t*>(img);
  const int head = blockIdx.y, b = head / a.hkv, h = head % a.hkv;
  const int tid = threadIdx.x;
  // this sequence's tokens of the call: [t0, t1)
  const int64_t len = a.sm.len(b, a.cap);
  const int64_t t0 = a.sm.tail ? max((int64_t)0, len - a.n) : a.t0;
  const int64_t t1 = a.sm.tail ? len : min(a.t0 + a.n, len);
  if (t1 <= t0) return;

  if (tid == 0) {
    s.meta = a.meta[head];
    s.overflow = 0;
  }
  for (int i = tid; i < kThrEntries; i += kQThreads) s.thr[i] = a.thr[i];
  const float* mr = a.mrow + (size_t)head * kD * kD;
  for (int idx = tid; idx < kD * kD; idx += kQThreads) {
    const int r = idx / kD, d = idx % kD;
    s.mt[d][r] = mr[idx];
    s.rt[d][r] = a.rot_v[idx];
  }
  __syncthreads();
  const HeadMeta& m = s.meta;
  const T* kbase = reinterpret_cast<const T*>(a.k) + b * a.s0 + h * a.s1;
  const T* vbase = reinterpret_cast<const T*>(a.v) + b * a.s0 + h * a.s1;
  const int vcode_off = 1024 * a.kb, vnorm_off = value_norm_offset(a.kb, a.vb);
  const int knorm_off = key_norm_offset(a.kb, a.vb);
  const int64_t tile_first = t0 / kTile, tile_last = (t1 - 1) / kTile;
  const int tb = tid >> 4, rb = tid & 15;
  const float sqrt_d = sqrtf((float)kD);

  for (int64_t tile = tile_first + blockIdx.x; tile <= tile_last; tile += gridDim.x) {
    const int64_t tok0 = tile * kTile;
    const bool full = tok0 >= t0 && tok0 + kTile <= t1;
    uint8_t* gimg = a.sm.tile(a.packed, head, tile);
    for (int i = tid; i < a.tile_bytes / 16; i += kQThreads)
      reinterpret_cast<uint4*>(img)[i] =
          full ? make_uint4(0, 0, 0, 0) : reinterpret_cast<const uint4*>(gimg)[i];
    // ------------------------------------------------------------------- keys
    load_tile<T>(s, kbase, tok0, t0, t1 - t0, a.s2);
    __syncthreads();
    for (int task = tid; task < kTile * m.n_groups; task += kQThreads) {
      const int j = task % kTile, g = task / kTile;
      const int64_t t = tok0 + j;
      double acc = 0.0;
      for (int blk = 0; blk < kBlocks; ++blk) {
        if (m.block_group[blk] != g) continue;
        const int p0 = a.pairing == GTQ_PAIRING_HALF ? blk : 2 * blk;
        const int p1 = a.pairing == GTQ_PAIRING_HALF ? blk + kBlocks : 2 * blk + 1;
        const double x0 = s.x[p0][j], x1 = s.x[p1][j];
        acc += x0 * x0;
        acc += x1 * x1;
      }
      const double nrm = sqrt(acc);
      s.scale[j][g] = nrm > 0.0 ? (float)((double)m.sqrt_m[g] / nrm) : 0.f;
      if (t >= t0 && t < t1) {
        int ovf = 0;
        const __half hn = norm_to_half(nrm, &ovf);
        if (ovf) s.overflow = 1;
        reinterpret_cast<__half*>(img + knorm_off + g * 128)[(j & 7) * 8 + (j >> 3)] = hn;
      }
    }
    __syncthreads();
    {
      float y[4][8];
      small_gemm(s.mt, s.x, tb, rb, y);
#pragma unroll
      for (int a2 = 0; a2 < 4; ++a2) {
        const int j = 4 * tb + a2;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int pos = 8 * rb + c, slot = pos >> 1;
          uint8_t code = 0;
          if (slot < m.n_slots) {
            const int g = m.slot_group[slot];
            const float sc = s.scale[j][g];
            if (sc != 0.f) code = (uint8_t)lm_code(y[a2][c] * sc, s.thr, m.slot_width[slot]);
          }
          s.codes[j][pos] = code;
        }
      }
    }
    __syncthreads();
    // pack keys: one thread per slot (all 8 portions, 16 w bytes, 16-byte aligned)
    for (int slot = tid; slot < m.n_slots; slot += kQThreads) {
      const int w = m.slot_width[slot];
      uint32_t* base = img32 + m.slot_koff[slot] / 4;
      for (int g = 0; g < 8; ++g)
        for (int u = 0; u < 8; ++u) {
          const int j = g + 8 * u;
          const int64_t t = tok0 + j;
          if (t < t0 || t >= t1) continue;
          for (int e = 0; e < 2; ++e)
            put_bits(base, g * 16 * w + (2 * u + e) * w, s.codes[j][2 * slot + e], w);
        }
    }
    __syncthreads();
    // ----------------------------------------------------------------- values
    if (a.vb == 0) {  // K-only: the tile holds keys only
      for (int i = tid; i < a.tile_bytes / 16; i += kQThreads)
        reinterpret_cast<uint4*>(gimg)[i] = reinterpret_cast<const uint4*>(img)[i];
      __syncthreads();
      continue;
    }
    load_tile<T>(s, vbase, tok0, t0, t1 - t0, a.s2);
    __syncthreads();
    if (tid < kTile) {
      const int j = tid;
      const int64_t t = tok0 + j;
      double acc = 0.0;
      for (int d = 0; d < kD; ++d) {
        const double x = s.x[d][j];
        acc += x * x;
      }
      const double nrm = sqrt(acc);
      s.scale[j][0] = nrm > 0.0 ? (float)((double)sqrt_d / nrm) : 0.f;
      if (t >= t0 && t < t1) {
        int ovf = 0;
        const __half hn = norm_to_half(nrm, &ovf);
        if (ovf) s.overflow = 1;
        reinterpret_cast<__half*>(img + vnorm_off)[(j & 7) * 8 + (j >> 3)] = hn;
      }
    }
    __syncthreads();
    {
      float y[4][8];
      small_gemm(s.rt, s.x, tb, rb, y);
#pragma unroll
      for (int a2 = 0; a2 < 4; ++a2) {
        const int j = 4 * tb + a2;
        const float sc = s.scale[j][0];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          s.codes[j][8 * rb + c] = sc != 0.f ? (uint8_t)lm_code(y[a2][c] * sc, s.thr, a.vb) : 0;
      }
    }
    __syncthreads();
    // pack values: one thread per portion (i, g, c): 32 codes, 4 vb bytes
    {
      const int p = tid, i = p >> 5, g = (p >> 2) & 7, c = p & 3;
      uint32_t* base = img32 + (vcode_off + p * 4 * a.vb) / 4;
      for (int x = 0; x < 32; ++x) {
        const int dim = 16 * i + g + 8 * ((x >> 1) & 1);
        const int j = 16 * (x >> 3) + 2 * c + (x & 1) + 8 * ((x >> 2) & 1);
        const int64_t t = tok0 + j;
        if (t < t0 || t >= t1) continue;
        put_bits(base, x * a.vb, s.codes[j][dim], a.vb);
      }
    }
    __syncthreads();
    for (int i = tid; i < a.tile_bytes / 16; i += kQThreads)
      reinterpret_cast<uint4*>(gimg)[i] = reinterpret_cast<const uint4*>(img)[i];
    __syncthreads();
  }
  if (tid == 0 && s.overflow) atomicOr(a.status, kStatusOverflow);
}

}  // namespace

cudaError_t launch_quantize_cc(const gtq_plan* p, const void* k, const void* v, const int64_t* st,
                               int64_t t0, int64_t n, uint8_t* packed, const SeqMap& sm,
                               cudaStream_t s) {
  QuantArgs a;
  a.k = k; a.v = v;
  a.s0 = st[0]; a.s1 = st[1]; a.s2 = st[2];
  a.t0 = t0; a.n = n;
  a.packed = packed;
  a.meta = p->d_meta;
  a.mrow = p->d_mrow;
  a.rot_v = p->tab.rot_v;
  a.thr = p->tab.thr;
  a.hkv = p->cfg.n_kv_heads;
  a.pairing = p->cfg.rope_pairing;
  a.n_tiles = p->n_tiles;
  a.tile_bytes = (int)p->tile_bytes;
  a.kb = p->cfg.k_bits;
  a.vb = p->cfg.v_bits;
  a.status = p->d_status;
  a.sm = sm;
  a.cap = p->cfg.t_capacity;
  const size_t smem = kImgOffset + p->tile_bytes;
  const int64_t tiles = sm.tail ? (n + kTile - 1) / kTile + 1 : (t0 + n - 1) / kTile - t0 / kTile + 1;
  int per_head = (int)std::min<int64_t>(tiles, std::max(1, (p->n_sms + p->n_heads - 1) / p->n_heads));
  dim3 grid(per_head, p->n_heads);
  cudaError_t e;
  if (p->cfg.in_dtype == GTQ_DTYPE_FP16) {
    e = cudaFuncSetAttribute(quantize_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    quantize_kernel<__half><<<grid, kQThreads, smem, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(quantize_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    quantize_kernel<float><<<grid, kQThreads, smem, s>>>(a);
  }
  return cudaGetLastError();
}

// Whole 128-token tiles of fp16 inputs go to the tensor-core kernel; the ragged
// edges (partial packed tiles, appends) and fp32 inputs to the CUDA-core kernel.
// Tokens [t0, t0 + n) outside the tensor-core tiles: a few tokens (a
// decode-time append) go to the append kernel, more to the CUDA-core kernel.
static cudaError_t launch_edge(const gtq_plan* p, const void* k, const void* v, const int64_t* st,
                               int64_t t0, int64_t n, uint8_t* packed, const SeqMap& sm,
                               cudaStream_t s) {
  if (n <= kAppendMax) return launch_append(p, k, v, st, t0, n, packed, sm, s);
  return launch_quantize_cc(p, k, v, st, t0, n, packed, sm, s);
}

cudaError_t launch_quantize(const gtq_plan* p, const void* k, const void* v, const int64_t* st,
                            int64_t t0, int64_t n, uint8_t* packed, const SeqMap& sm,
                            cudaStream_t s) {
  if (sm.tail) return launch_edge(p, k, v, st, 0, n, packed, sm, s);  // starts per sequence
  if (p->cfg.in_dtype == GTQ_DTYPE_FP16 && p->cfg.head_dim == kD) {
    const int64_t mt0 = (t0 + 127) / 128, mt1 = (t0 + n) / 128;
    if (mt1 > mt0) {
      cudaError_t e = launch_quantize_tc(p, k, v, st, mt0, mt1, packed, sm, s);
      if (e != cudaErrorNotSupported) {
        if (e != cudaSuccess) return e;
        if (mt0 * 128 > t0) e = launch_edge(p, k, v, st, t0, mt0 * 128 - t0, packed, sm, s);
        if (e == cudaSuccess && t0 + n > mt1 * 128)
          e = launch_edge(p, k, v, st, mt1 * 128, t0 + n - mt1 * 128, packed, sm, s);
        return e;
      }
    }
  }
  return launch_edge(p, k, v, st, t0, n, packed, sm, s);
}

}  // namespace gtq
