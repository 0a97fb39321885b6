// Block-GTQ allocation on the device ("RoPE-Aware Bit Allocation for KV-Cache
// Quantization", Abstract): per layer and KV head, an energy score of every
// RoPE block that needs no labels, then integer widths given one bit at a time
// to the block with the largest marginal gain.
//
//   energy_partial_kernel  E partial sums over token chunks, fp64, fixed order
//   energy_finish_kernel   E_i = (sum over p0 and p1 of block i) / T
//   greedy_kernel          one warp per head: +1 bit to argmax E_i (D(b_i) - D(b_i+1)),
//                          ties to the lower index, until sum 2 b_i = k_bits * d
//   meta_kernel            groups (descending width), slots, decode segments and
//                          the per-head key rotation rows M_h in packed order
#include <cmath>
#include <cstdio>
#include <mutex>

#include "gtq_internal.h"

namespace gtq {
namespace {

constexpr int kEnergyChunk = 1024;  // tokens per energy CTA

template <typename T>
__device__ inline void load8(const T* p, float (&x)[8]);
template <>
__device__ inline void load8<__half>(const __half* p, float (&x)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
template <>
__device__ inline void load8<float>(const float* p, float (&x)[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// grid (chunks, heads), 256 threads = 16 token lanes x 16 dim lanes (8 dims each)
template <typename T>
__global__ void __launch_bounds__(256) energy_partial_kernel(const T* __restrict__ k, int64_t s0,
                                                             int64_t s1, int64_t s2, int hkv,
                                                             int d, int64_t T_tok,
                                                             const int32_t* __restrict__ seq_lens,
                                                             double* __restrict__ part) {
  const int head = blockIdx.y, b = head / hkv, h = head % hkv;
  const int tl = threadIdx.x >> 4, dl = threadIdx.x & 15;
  const int64_t T_b = seq_lens ? max((int64_t)0, min((int64_t)seq_lens[b], T_tok)) : T_tok;
  const int64_t t_begin = (int64_t)blockIdx.x * kEnergyChunk;
  const int64_t t_end = min(t_begin + kEnergyChunk, T_b);
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
  const bool active = dl * 8 < d;
  if (active) {
    const T* base = k + b * s0 + h * s1 + dl * 8;
    for (int64_t t = t_begin + tl; t < t_end; t += 16) {
      float x[8];
      load8<T>(base + t * s2, x);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += (double)x[i] * (double)x[i];  // exact squares
    }
  }
  __shared__ double red[16][128];
#pragma unroll
  for (int i = 0; i < 8; ++i) red[tl][dl * 8 + i] = acc[i];
  __syncthreads();
  if (threadIdx.x < 128 && threadIdx.x < d) {
    double s = 0.0;
    for (int j = 0; j < 16; ++j) s += red[j][threadIdx.x];  // fixed order
    part[((size_t)head * gridDim.x + blockIdx.x) * 128 + threadIdx.x] = s;
  }
}

// grid heads, 64 threads (one per block)
__global__ void energy_finish_kernel(const double* __restrict__ part, int chunks, int d,
                                     int pairing, int64_t T_tok, const int32_t* __restrict__ seq_lens,
                                     int hkv, double* __restrict__ energy) {
  const int head = blockIdx.x, i = threadIdx.x, nb = d / 2;
  if (i >= nb) return;
  const int64_t T_b =
      seq_lens ? max((int64_t)0, min((int64_t)seq_lens[head / hkv], T_tok)) : T_tok;
  const int p0 = pairing == GTQ_PAIRING_HALF ? i : 2 * i;
  const int p1 = pairing == GTQ_PAIRING_HALF ? i + nb : 2 * i + 1;
  double s0 = 0.0, s1 = 0.0;
  for (int c = 0; c < chunks; ++c) {
    s0 += part[((size_t)head * chunks + c) * 128 + p0];
    s1 += part[((size_t)head * chunks + c) * 128 + p1];
  }
  energy[(size_t)head * nb + i] = T_b > 0 ? (s0 + s1) / (double)T_b : 0.0;
}

// one warp per head
__global__ void greedy_kernel(const double* __restrict__ energy, const double* __restrict__ dist,
                              int nb, int k_bits, int max_bits, int n_heads,
                              uint8_t* __restrict__ bits) {
  const int head = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (head >= n_heads) return;
  double dd[GTQ_MAX_BITS + 2];
#pragma unroll
  for (int i = 0; i <= GTQ_MAX_BITS; ++i) dd[i] = dist[i];
  dd[GTQ_MAX_BITS + 1] = dd[GTQ_MAX_BITS];
  const int i0 = lane, i1 = lane + 32;
  const double e0 = i0 < nb ? energy[(size_t)head * nb + i0] : 0.0;
  const double e1 = i1 < nb ? energy[(size_t)head * nb + i1] : 0.0;
  int b0 = 0, b1 = 0;
  const int steps = k_bits * nb;  // sum b_i = k_bits * d / 2
  for (int s = 0; s < steps; ++s) {
    double g0 = -1.0, g1 = -1.0;
    if (i0 < nb && b0 < max_bits) g0 = e0 * (dd[b0] - dd[b0 + 1]);
    if (i1 < nb && b1 < max_bits) g1 = e1 * (dd[b1] - dd[b1 + 1]);
    double g = g0;
    int idx = i0;
    if (g1 > g0) { g = g1; idx = i1; }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      double og = __shfl_xor_sync(0xffffffffu, g, off);
      int oi = __shfl_xor_sync(0xffffffffu, idx, off);
      if (og > g || (og == g && oi < idx)) { g = og; idx = oi; }
    }
    if (idx == i0) ++b0;
    if (idx == i1) ++b1;
  }
  if (i0 < nb) bits[(size_t)head * nb + i0] = (uint8_t)b0;
  if (i1 < nb) bits[(size_t)head * nb + i1] = (uint8_t)b1;
}

// one CTA (128 threads) per head; head_dim 128 only
__global__ void __launch_bounds__(128) meta_kernel(const uint8_t* __restrict__ bits,
                                                   const double* __restrict__ energy,
                                                   const double* __restrict__ rot_k, int pairing,
                                                   HeadMeta* __restrict__ meta_out,
                                                   float* __restrict__ mrow,
                                                   float* __restrict__ rotpack) {
  const int head = blockIdx.x;
  __shared__ HeadMeta m;
  __shared__ uint8_t grp_blocks[kMaxGroups][kBlocks];
  __shared__ int grp_count[kMaxGroups];
  if (threadIdx.x == 0) {
    const uint8_t* bb = bits + (size_t)head * kBlocks;
    const double* ee = energy + (size_t)head * kBlocks;
    int ng = 0, slot = 0, koff = 0;
    double gen[kMaxGroups];
    for (int i = 0; i < kBlocks; ++i) m.block_group[i] = 0xFF;
    for (int w = GTQ_MAX_BITS; w >= 1; --w) {
      int cnt = 0;
      double eg = 0.0;
      for (int i = 0; i < kBlocks; ++i)
        if (bb[i] == w) {
          grp_blocks[ng][cnt++] = (uint8_t)i;
          m.block_group[i] = (uint8_t)ng;
          eg += ee[i];
        }
      if (!cnt) continue;
      grp_count[ng] = cnt;
      gen[ng] = eg;
      m.grp_width[ng] = (uint8_t)w;
      m.grp_m[ng] = (uint8_t)(2 * cnt);
      m.grp_first_slot[ng] = (uint8_t)slot;
      m.sqrt_m[ng] = (float)sqrt(2.0 * cnt);
      m.inv_sqrt_m[ng] = (float)(1.0 / sqrt(2.0 * cnt));
      for (int s = 0; s < cnt; ++s, ++slot) {
        m.slot_width[slot] = (uint8_t)w;
        m.slot_group[slot] = (uint8_t)ng;
        m.slot_koff[slot] = (uint16_t)koff;
        koff += 16 * w;
      }
      ++ng;
    }
    for (int s = slot; s < kBlocks; ++s) {
      m.slot_width[s] = 0;
      m.slot_group[s] = 0xFF;
      m.slot_koff[s] = (uint16_t)koff;
    }
    for (int g = ng; g < kMaxGroups; ++g) {
      m.grp_width[g] = 0; m.grp_m[g] = 0; m.grp_first_slot[g] = (uint8_t)slot;
      m.sqrt_m[g] = 0.f; m.inv_sqrt_m[g] = 0.f; grp_count[g] = 0; gen[g] = 0.0;
    }
    m.n_groups = ng;
    m.n_slots = slot;
    // split rule: widest groups first until the unsplit rest holds <= 1/4 of the energy
    double tot = 0.0;
    for (int g = 0; g < ng; ++g) tot += gen[g];
    double rem = tot;
    for (int g = 0; g < kMaxGroups; ++g) {
      m.grp_split[g] = 0;
      if (g < ng && rem > 0.25 * tot) {
        m.grp_split[g] = 1;
        rem -= gen[g];
      }
    }
    // decode k-tiles: each group's slots in runs of at most 8 (one mma k-step of 16 coords)
    int nk = 0;
    for (int g = 0; g < kMaxGroups; ++g) m.grp_kt0[g] = m.grp_kt1[g] = 0;
    for (int g = 0; g < ng; ++g) {
      const int first = m.grp_first_slot[g], cnt = grp_count[g];
      m.grp_kt0[g] = (uint8_t)nk;
      m.grp_kt1[g] = (uint8_t)(nk + (cnt + 7) / 8);
      for (int off = 0; off < cnt; off += 8) {
        m.kt_group[nk] = (uint8_t)g;
        m.kt_first_slot[nk] = (uint8_t)(first + off);
        m.kt_nslots[nk] = (uint8_t)min(8, cnt - off);
        m.kt_flags[nk] = (uint8_t)((off == 0 ? 1 : 0) | (off + 8 >= cnt ? 2 : 0));
        ++nk;
      }
    }
    for (int k = nk; k < kMaxKt; ++k) {
      m.kt_group[k] = 0; m.kt_first_slot[k] = 0; m.kt_nslots[k] = 0; m.kt_flags[k] = 0;
    }
    m.n_ktiles = nk;
    m.reserved = 0;
  }
  __syncthreads();
  // key rotation rows: M_h[pos][dim], pos = 2 * slot + e  <->  row r = 2 (slot - first) + e of R_m;
  // the rotation pack: coord_dim[pos] and every group's R_m transposed
  const int pos = threadIdx.x;
  float* row = mrow + ((size_t)head * kD + pos) * kD;
  float* pack = rotpack + (size_t)head * kRotPackMaxWords;
  uint8_t* coord_dim = reinterpret_cast<uint8_t*>(pack);
  for (int dd = 0; dd < kD; ++dd) row[dd] = 0.f;
  const int slot = pos >> 1;
  uint8_t cdim = 0;
  if (slot < m.n_slots) {
    const int g = m.slot_group[slot];
    const int mm = m.grp_m[g];
    const int r = 2 * (slot - m.grp_first_slot[g]) + (pos & 1);
    size_t off = 0;
    for (int q = 2; q < mm; q += 2) off += (size_t)q * q;
    const double* R = rot_k + off + (size_t)r * mm;
    size_t poff = kRotPackHeaderWords;  // this group's block in the pack
    for (int gg = 0; gg < g; ++gg) poff += (size_t)m.grp_m[gg] * m.grp_m[gg];
    for (int c = 0; c < mm; ++c) {
      const int blk = grp_blocks[g][c >> 1], el = c & 1;
      const int dim = pairing == GTQ_PAIRING_HALF ? blk + el * kBlocks : 2 * blk + el;
      row[dim] = (float)R[c];
      pack[poff + (size_t)c * mm + r] = (float)R[c];
    }
    // coordinate r of the group (the same index range as its rows) has this dim
    const int blk = grp_blocks[g][r >> 1], el = r & 1;
    cdim = (uint8_t)(pairing == GTQ_PAIRING_HALF ? blk + el * kBlocks : 2 * blk + el);
  }
  coord_dim[pos] = cdim;
  if (threadIdx.x == 0) meta_out[head] = m;
}

}  // namespace

cudaError_t launch_energy(const gtq_plan* p, const void* k, int64_t T, const int64_t* st,
                          const int32_t* seq_lens, cudaStream_t s) {
  const int chunks = (int)((T + kEnergyChunk - 1) / kEnergyChunk);
  double* part = nullptr;
  cudaError_t e = cudaMallocAsync((void**)&part, (size_t)p->n_heads * chunks * 128 * sizeof(double), s);
  if (e != cudaSuccess) return e;
  dim3 grid(chunks, p->n_heads);
  const int d = p->cfg.head_dim;
  if (p->cfg.in_dtype == GTQ_DTYPE_FP16)
    energy_partial_kernel<__half><<<grid, 256, 0, s>>>((const __half*)k, st[0], st[1], st[2],
                                                       p->cfg.n_kv_heads, d, T, seq_lens, part);
  else
    energy_partial_kernel<float><<<grid, 256, 0, s>>>((const float*)k, st[0], st[1], st[2],
                                                      p->cfg.n_kv_heads, d, T, seq_lens, part);
  energy_finish_kernel<<<p->n_heads, 64, 0, s>>>(part, chunks, d, p->cfg.rope_pairing, T,
                                                 seq_lens, p->cfg.n_kv_heads, p->d_energy);
  e = cudaGetLastError();
  cudaFreeAsync(part, s);
  return e;
}

cudaError_t launch_greedy_and_meta(const gtq_plan* p, cudaStream_t s) {
  const int warps = 4;
  greedy_kernel<<<(p->n_heads + warps - 1) / warps, 32 * warps, 0, s>>>(
      p->d_energy, p->tab.dist, p->n_blocks, p->cfg.k_bits, p->cfg.max_bits, p->n_heads,
      p->d_bits);
  if (p->cfg.head_dim == kD) {
    meta_kernel<<<p->n_heads, 128, 0, s>>>(p->d_bits, p->d_energy, p->tab.rot_k,
                                           p->cfg.rope_pairing, p->d_meta, p->d_mrow, p->d_rotpack);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return build_b_images(p->d_mrow, p->n_heads, (size_t)kD * kD, p->d_bimg, s);
  }
  return cudaGetLastError();
}

}  // namespace gtq

namespace gtq {

// ---------------------------------------------------------------------------
// Energy pass without any device allocation.
//
// gtq_alloc_bits gets its energy-pass scratch (fp64 partial sums per token
// chunk) from cudaMallocAsync.  Some callers cannot allocate device memory at
// call time: code that runs while a CUDA graph is being captured, servers that
// reserve all device memory up front and forbid later allocations, and
// real-time loops that cannot afford an allocator call.  gtq_block_energy_noalloc
// runs the same two kernels with that scratch in the fixed array below instead.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocEnergyDoubles = (size_t)1 << 19;  // 4 MiB of partial sums per GPU

// One copy per GPU that loads the library, alive until the process exits.
static __device__ __align__(256) double g_energy_scratch[kNoAllocEnergyDoubles];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
double* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_energy_scratch on `device` (the current device); looked up
// once per device.  In host code the array's name is only a host-side stand-in.
cudaError_t scratch_for(int device, double** out) {
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (!g_scratch_ptr[device]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_energy_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[device] = static_cast<double*>(p);
  }
  *out = g_scratch_ptr[device];
  return cudaSuccess;
}

}  // namespace
}  // namespace gtq

extern "C" int gtq_block_energy_noalloc(const gtq_config* cfg, const void* k_dev, int64_t T,
                                        const int64_t k_strides[4], double* energy_dev,
                                        void* stream) {
  using namespace gtq;
  if (!cfg || !k_dev || !k_strides || !energy_dev) return GTQ_ERR_INVALID;
  if (cfg->batch < 1 || cfg->n_kv_heads < 1) return GTQ_ERR_INVALID;
  if (cfg->head_dim < 8 || cfg->head_dim > kD || (cfg->head_dim % 8)) return GTQ_ERR_UNSUPPORTED;
  if (cfg->rope_pairing != GTQ_PAIRING_HALF && cfg->rope_pairing != GTQ_PAIRING_INTERLEAVED)
    return GTQ_ERR_INVALID;
  if (cfg->in_dtype != GTQ_DTYPE_FP16 && cfg->in_dtype != GTQ_DTYPE_FP32) return GTQ_ERR_INVALID;
  if (T < 1) return GTQ_ERR_INVALID;
  const int esz = cfg->in_dtype == GTQ_DTYPE_FP16 ? 2 : 4;
  if (k_strides[3] != 1 || ((uintptr_t)k_dev % 16) || ((uintptr_t)energy_dev % 8))
    return GTQ_ERR_INVALID;
  for (int i = 0; i < 3; ++i)
    if (k_strides[i] < 0 || (k_strides[i] * esz) % 16) return GTQ_ERR_INVALID;
  // heads is grid.y of both kernels: the product is formed in 64 bits and
  // bounded by the grid limit before anything else uses it
  const int64_t heads64 = (int64_t)cfg->batch * (int64_t)cfg->n_kv_heads;
  if (heads64 > 65535) {
    set_last_error("gtq_block_energy_noalloc: batch * n_kv_heads exceeds 65535");
    return GTQ_ERR_INVALID;
  }
  const int heads = (int)heads64;
  const int64_t chunks = (T + kEnergyChunk - 1) / kEnergyChunk;
  if (chunks > (int64_t)kNoAllocEnergyDoubles ||
      heads64 * chunks * 128 > (int64_t)kNoAllocEnergyDoubles) {
    char msg[160];
    snprintf(msg, sizeof(msg),
             "gtq_block_energy_noalloc: %d heads x %lld token chunks need %lld partial sums, "
             "the fixed scratch holds %zu",
             heads, (long long)chunks, (long long)(heads64 * chunks * 128), kNoAllocEnergyDoubles);
    set_last_error(msg);
    return GTQ_ERR_UNSUPPORTED;
  }
  int device = 0;
  double* part = nullptr;
  cudaError_t e = cudaGetDevice(&device);
  if (e == cudaSuccess) e = scratch_for(device, &part);
  if (e != cudaSuccess) return record_cuda_error(e);
  cudaStream_t s = (cudaStream_t)stream;
  dim3 grid((unsigned)chunks, heads);
  // every partial sum read by energy_finish_kernel is first written by
  // energy_partial_kernel, so the shared scratch needs no clearing
  if (cfg->in_dtype == GTQ_DTYPE_FP16)
    energy_partial_kernel<__half><<<grid, 256, 0, s>>>((const __half*)k_dev, k_strides[0],
                                                       k_strides[1], k_strides[2],
                                                       cfg->n_kv_heads, cfg->head_dim, T, nullptr,
                                                       part);
  else
    energy_partial_kernel<float><<<grid, 256, 0, s>>>((const float*)k_dev, k_strides[0],
                                                      k_strides[1], k_strides[2],
                                                      cfg->n_kv_heads, cfg->head_dim, T, nullptr,
                                                      part);
  energy_finish_kernel<<<heads, 64, 0, s>>>(part, (int)chunks, cfg->head_dim, cfg->rope_pairing,
                                            T, nullptr, cfg->n_kv_heads, energy_dev);
  return record_cuda_error(cudaGetLastError());
}
