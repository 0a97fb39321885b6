// Decode-time append: TurboQuant-MSE coding of a few new tokens (n <= 16 per
// call) into an existing packed cache under the allocation already in the
// plan ("RoPE-Aware Bit Allocation for KV-Cache Quantization", Abstract: the
// widths are chosen per layer and KV head, and decoding then runs from the
// packed cache, which a serving loop extends one token at a time).
//
// One CTA of 128 threads per (head, role): role 0 codes the keys, role 1 the
// values.  The role's rotation (the key groups' blocks, or R_V^T) arrives in
// shared memory by one bulk copy while the new rows load; thread p then owns
// rotated coordinate p (packed position p for keys, row p of R_V for values)
// for all new tokens at once:
//   keys    y_p = sum_c R_g[r][c] k[dim(c)] over the group's m coordinates
//           (the plan's rotation pack: R_g transposed, so that the threads of
//           a group read consecutive words), group norms in fp64 by one warp
//           per group in a fixed order;
//   values  y_r = sum_d R_V[r][d] v[d] (R_V^T: consecutive threads, consecutive
//           words), the norm in fp64 by one warp.
// Codes are the number of fp32 thresholds below y * sqrt(m) / n (0 for a zero
// vector).  Each code is written into the packed tile by an atomic AND that
// clears its bits and an atomic OR that sets them, so codes of other tokens
// that share the words are left as they are; norms are plain fp16 stores.
#include "gtq_internal.h"

namespace gtq {
namespace {

constexpr int kAThreads = 128;
constexpr int kRotBytes = (int)kRotPackBytes;  // >= R_V^T (64 KB)
constexpr uint64_t kAWaitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
// bounded wait on phase 0 of an mbarrier; false after about two seconds
__device__ bool wait_phase0(uint64_t* bar) {
  uint64_t t0 = 0;
  for (unsigned i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar))
        : "memory");
    if (ok) return true;
    if ((i & 63u) == 63u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0)
        t0 = now;
      else if (now - t0 > kAWaitNs)
        return false;
    }
  }
}

struct AppendArgs {
  const void* k;
  const void* v;
  int64_t s0, s1, s2;
  int64_t t0;
  int n;
  uint8_t* packed;
  const HeadMeta* meta;
  const float* rotpack;  // [heads][kRotPackMaxWords]
  const float* rot_vt;   // R_V^T
  const float* thr;      // fp32 thresholds, width w at thr_base(w)
  int hkv;
  int64_t n_tiles;
  int tile_bytes;
  int kb, vb;
  int* status;
  SeqMap sm;
  int64_t cap;
};

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<__half>(const __half* p) { return __half2float(*p); }
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return *p; }

// number of width-w thresholds strictly below y (binary search, ascending thresholds)
__device__ __forceinline__ uint32_t lm_code(float y, const float* thr, int w) {
  const float* t = thr + thr_base(w);
  int lo = 0;
  for (int step = 1 << (w - 1); step; step >>= 1)
    if (y > t[lo + step - 1]) lo += step;
  return (uint32_t)lo;
}

// write the w-bit code at bit offset `bit` of the tile, leaving other bits alone
__device__ __forceinline__ void put_code(uint8_t* tile, uint32_t bit, uint32_t code, int w) {
  uint32_t* words = reinterpret_cast<uint32_t*>(tile);
  const uint32_t wd = bit >> 5, sh = bit & 31;
  const uint64_t mask = ((1ull << w) - 1ull) << sh;
  const uint64_t val = ((uint64_t)code << sh) & mask;
  atomicAnd(&words[wd], ~(uint32_t)mask);
  atomicOr(&words[wd], (uint32_t)val);
  if (sh + (uint32_t)w > 32) {
    atomicAnd(&words[wd + 1], ~(uint32_t)(mask >> 32));
    atomicOr(&words[wd + 1], (uint32_t)(val >> 32));
  }
}

__device__ __forceinline__ __half norm_half(double n, int* ovf) {
  if (n > 65504.0) {
    *ovf = 1;
    n = 65504.0;
  }
  return __double2half(n);  // round-to-nearest-even from fp64
}

template <typename T>
__global__ void __launch_bounds__(kAThreads) append_kernel(AppendArgs a) {
  extern __shared__ __align__(16) float rot[];  // the role's rotation, kRotBytes
  __shared__ float x[kAppendMax][kD];           // the new tokens' K or V rows
  __shared__ float thr[kThrEntries];
  __shared__ double nrm[kAppendMax][kMaxGroups];
  __shared__ HeadMeta m;
  __shared__ __align__(8) uint64_t bar;
  __shared__ int ovf;
  const int head = blockIdx.x, role = blockIdx.y;
  const int b = head / a.hkv, h = head % a.hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Before the grid-dependency wait only the plan's constants are read (its
  // metadata, rotation blocks and thresholds, written when the plan was made);
  // the lengths, the new rows and the packed cache may come from the previous
  // grid and are read or written after it.
  if (tid == 0) {
    m = a.meta[head];
    ovf = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    int bytes = kD * kD * 4;
    const void* src = a.rot_vt;
    if (role == 0) {
      int words = kRotPackHeaderWords;
      for (int gi = 0; gi < m.n_groups; ++gi) words += (int)m.grp_m[gi] * m.grp_m[gi];
      bytes = (words * 4 + 15) & ~15;
      src = a.rotpack + (size_t)head * kRotPackMaxWords;
    }
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(&bar)),
                 "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(rot)),
        "l"(src), "r"(bytes), "r"(smem_u32(&bar))
        : "memory");
  }
  for (int i = tid; i < kThrEntries; i += kAThreads) thr[i] = a.thr[i];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // tokens of this sequence among the call's: [t0, t0 + n)
  const int64_t len = a.sm.len(b, a.cap);
  const int64_t t0 = a.sm.tail ? max((int64_t)0, len - a.n) : a.t0;
  const int n = (int)max((int64_t)0, min((int64_t)a.n, len - t0));
  if (n == 0) {  // nothing to write: only the rotation copy must land before the exit
    __syncthreads();
    if (tid == 0 && !wait_phase0(&bar)) atomicOr(a.status, kStatusTimeout);
    return;
  }
  const T* src = reinterpret_cast<const T*>(role == 0 ? a.k : a.v) + b * a.s0 + h * a.s1;
  for (int i = tid; i < n * kD; i += kAThreads) {
    const int j = i / kD, d = i % kD;
    x[j][d] = ld_f<T>(src + (t0 + j) * a.s2 + d);
  }
  __syncthreads();
  // every thread waits for the rotation (and so no copy outlives the CTA)
  if (!__syncthreads_and(wait_phase0(&bar))) {
    if (tid == 0) atomicOr(a.status, kStatusTimeout);
    return;
  }
  const int p = tid;

  if (role == 0) {
    // ---------------------------------------------------------------- keys
    const float* pack = rot;
    const uint8_t* coord_dim = reinterpret_cast<const uint8_t*>(pack);
    // group norms: one warp per group, lanes stride over the group's coordinates
    for (int gi = warp; gi < m.n_groups; gi += kAThreads / 32) {
      const int first = 2 * m.grp_first_slot[gi], mm = m.grp_m[gi];
      for (int j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int c = lane; c < mm; c += 32) {
          const double v = x[j][coord_dim[first + c] & (kD - 1)];
          acc = fma(v, v, acc);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) nrm[j][gi] = sqrt(acc);
      }
    }
    __syncthreads();
    const int slot = p >> 1;
    if (slot < m.n_slots) {
      const int gi = m.slot_group[slot], mm = m.grp_m[gi], w = m.slot_width[slot];
      const int first = 2 * m.grp_first_slot[gi], r = p - first;
      int off = kRotPackHeaderWords;
      for (int gg = 0; gg < gi; ++gg) off += (int)m.grp_m[gg] * m.grp_m[gg];
      float acc[kAppendMax];
#pragma unroll
      for (int j = 0; j < kAppendMax; ++j) acc[j] = 0.f;
      for (int c = 0; c < mm; ++c) {
        const float rv = pack[off + c * mm + r];
        const int d = coord_dim[first + c] & (kD - 1);
#pragma unroll
        for (int j = 0; j < kAppendMax; ++j)
          if (j < n) acc[j] = fmaf(rv, x[j][d], acc[j]);
      }
      const int e = p & 1;
#pragma unroll
      for (int j = 0; j < kAppendMax; ++j) {
        if (j >= n) break;
        const int64_t t = t0 + j;
        const int jj = (int)(t % kTile), g8 = jj & 7, u = jj >> 3;
        const double n = nrm[j][gi];
        const uint32_t code =
            n > 0.0 ? lm_code(acc[j] * (float)((double)m.sqrt_m[gi] / n), thr, w) : 0u;
        uint8_t* tile = a.sm.tile(a.packed, head, t / kTile);
        const uint32_t bit = 8u * (m.slot_koff[slot] + g8 * 2 * w) + (uint32_t)((2 * u + e) * w);
        put_code(tile, bit, code, w);
      }
    }
    // norms: thread (token j, group gi)
    const int knorm_off = key_norm_offset(a.kb, a.vb);
    for (int i = tid; i < n * m.n_groups; i += kAThreads) {
      const int j = i / m.n_groups, gi = i % m.n_groups;
      const int64_t t = t0 + j;
      const int jj = (int)(t % kTile);
      int o = 0;
      const __half hn = norm_half(nrm[j][gi], &o);
      if (o) ovf = 1;
      uint8_t* tile = a.sm.tile(a.packed, head, t / kTile);
      reinterpret_cast<__half*>(tile + knorm_off + gi * 128)[(jj & 7) * 8 + (jj >> 3)] = hn;
    }
  } else {
    // -------------------------------------------------------------- values
    for (int j = warp; j < n; j += kAThreads / 32) {
      double acc = 0.0;
      for (int d = lane; d < kD; d += 32) {
        const double v = x[j][d];
        acc = fma(v, v, acc);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) nrm[j][0] = sqrt(acc);
    }
    __syncthreads();
    float acc[kAppendMax];
#pragma unroll
    for (int j = 0; j < kAppendMax; ++j) acc[j] = 0.f;
    for (int d = 0; d < kD; ++d) {
      const float rv = rot[d * kD + p];  // R_V[p][d]
#pragma unroll
      for (int j = 0; j < kAppendMax; ++j)
        if (j < n) acc[j] = fmaf(rv, x[j][d], acc[j]);
    }
    const float sqrt_d = sqrtf((float)kD);
    const int i16 = p >> 4, g = p & 7, hd = (p >> 3) & 1;  // dim tile, row, upper half
    const int vcode_off = 1024 * a.kb, vnorm_off = value_norm_offset(a.kb, a.vb);
#pragma unroll
    for (int j = 0; j < kAppendMax; ++j) {
      if (j >= n) break;
      const int64_t t = t0 + j;
      const int jj = (int)(t % kTile);
      const double n = nrm[j][0];
      const uint32_t code = n > 0.0 ? lm_code(acc[j] * (float)((double)sqrt_d / n), thr, a.vb) : 0u;
      // portion (i, g, c) and code index x: token 16 kk + 2c + lt + 8 ht
      const int kk = jj >> 4, ht = (jj >> 3) & 1, c = (jj >> 1) & 3, lt = jj & 1;
      const int portion = (i16 * 8 + g) * 4 + c;
      const int xi = kk * 8 + ht * 4 + hd * 2 + lt;
      uint8_t* tile = a.sm.tile(a.packed, head, t / kTile);
      put_code(tile, 8u * (uint32_t)(vcode_off + portion * 4 * a.vb) + (uint32_t)(xi * a.vb), code,
               a.vb);
      if (p == 0) {
        int o = 0;
        const __half hn = norm_half(n, &o);
        if (o) ovf = 1;
        reinterpret_cast<__half*>(tile + vnorm_off)[(jj & 7) * 8 + (jj >> 3)] = hn;
      }
    }
  }
  __syncthreads();
  if (tid == 0 && ovf) atomicOr(a.status, kStatusOverflow);
}

}  // namespace

cudaError_t launch_append(const gtq_plan* p, const void* k, const void* v, const int64_t* st,
                          int64_t t0, int64_t n, uint8_t* packed, const SeqMap& sm, cudaStream_t s) {
  if (n < 1 || n > kAppendMax) return cudaErrorInvalidValue;
  AppendArgs a;
  a.k = k;
  a.v = v;
  a.s0 = st[0];
  a.s1 = st[1];
  a.s2 = st[2];
  a.t0 = t0;
  a.n = (int)n;
  a.packed = packed;
  a.meta = p->d_meta;
  a.rotpack = p->d_rotpack;
  a.rot_vt = p->tab.rot_vt;
  a.thr = p->tab.thr;
  a.hkv = p->cfg.n_kv_heads;
  a.n_tiles = p->n_tiles;
  a.tile_bytes = (int)p->tile_bytes;
  a.kb = p->cfg.k_bits;
  a.vb = p->cfg.v_bits;
  a.status = p->d_status;
  a.sm = sm;
  a.cap = p->cfg.t_capacity;
  const dim3 grid((unsigned)p->n_heads, p->cfg.v_bits > 0 ? 2 : 1);  // K-only: keys alone
  // programmatic dependent launch: the constant prologue overlaps the previous grid
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kAThreads);
  cfg.dynamicSmemBytes = kRotBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (p->cfg.in_dtype == GTQ_DTYPE_FP16) {
    e = cudaFuncSetAttribute(append_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kRotBytes);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, append_kernel<__half>, a);
  } else {
    e = cudaFuncSetAttribute(append_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kRotBytes);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, append_kernel<float>, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace gtq
