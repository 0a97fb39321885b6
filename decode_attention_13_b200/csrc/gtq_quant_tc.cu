// Tensor-core quantize-pack (fp16 K/V, head_dim 128): the per-token rotations
// run as tcgen05 GEMMs with fp32 accumulators in tensor memory ("RoPE-Aware Bit
// Allocation for KV-Cache Quantization", Abstract: Block-GTQ quantizes keys with
// TurboQuant-MSE as the base quantizer, whose coder rotates every normalised
// vector before scalar Lloyd-Max coding).  Stored values are those of the CUDA-core quantizer
// (gtq_quant.cu): per token and key group g, n = ||k_g||, code = number of fp32
// thresholds below (sqrt(m)/n) (M_h k)_j, fp16(n) stored; values likewise with
// one group of 128 and R_V.
//
// One launch; a CTA works on one head in one role, keys or values (about two
// thirds of a head's CTAs take keys, whose tiles cost more; with many heads,
// 2u key and u value CTAs per head that run in waves), and walks the 128-token
// tiles that lie inside the tokens being written.  Per tile:
//   * code GEMM   D_c[coord][token] = R . X^T with R = M_h (keys) or R_V (values)
//                 split into fp16 hi + lo parts (A operand, resident in shared
//                 memory) and X the fp16 tile (B operand, TMA, 128B swizzle);
//                 two tensor-memory accumulators of 128 columns.
//   * gather GEMM D_p[token][row] = X . P^T with P a 0/1 matrix that lists the
//                 dims of key group 0, then group 1, ... (each group padded to 8
//                 rows); every output is one input element, so D_p holds the
//                 exact fp16 inputs as fp32, grouped by key group.  Keys only:
//                 the value norms are summed straight from the fp16 tile in
//                 shared memory.
// Warps: 0 TMA producer; 1 tensor-memory owner and MMA issuer; 2-5 norm warps
// (thread = token: group sums of squares from D_p); 6-13 code warps (thread =
// rotated coordinate, 64 tokens: codes, bit packing in registers with one
// partner lane, 8-byte stores straight into the packed tiles).
//
// Norms: the fp32 sum of exact squares has a rigorous relative error bound;
// when fp16 rounding of every value inside the bound agrees, that is the stored
// norm, otherwise (about 0.1-0.4 % of norms) the warp decides it exactly from the
// fp64 sum of squares of the fp16 tile in shared memory.  Scales for the codes
// come from the same sum (approximate reciprocal root).  A tile that holds a zero
// vector or group is flagged, and its codes are masked to 0.
// Waits suspend the thread (mbarrier try_wait with a time hint) and are bounded;
// on expiry the status word gets GTQ_ERR_TIMEOUT's bit.
#include <cuda.h>

#include <cmath>
#include <cstring>

#include "gtq_internal.h"

namespace gtq {
namespace {

constexpr int kTcWarps = 14;
constexpr int kTcThreads = 32 * kTcWarps;
constexpr int kMTile = 128;          // tokens per MMA tile (= 2 packed tiles)
constexpr int kStages = 3;           // input tile stages
constexpr uint32_t kSuspendHintNs = 1000000;  // mbarrier try_wait suspend-time hint
constexpr int kKeyShare = 67;        // percent of a head's CTAs that quantize keys
constexpr uint64_t kTcWaitNs = 2000000000ull;  // bound of every barrier wait

constexpr int kMaxPRows = 176;       // 128 dims + at most 6 padding rows for each of 8 groups
constexpr int kMaxChunks = kMaxPRows / 8;
constexpr int kScaleStride = 132;    // floats per (buffer, group) row of the scale table

constexpr uint32_t kBBytes = 65536;      // R image: hi 32 KB, lo 32 KB
constexpr uint32_t kStageBytes = 32768;  // X tile: 2 atoms x 128 rows x 128 B
constexpr uint32_t kOffB = 0;
constexpr uint32_t kOffP = kOffB + kBBytes;
constexpr uint32_t kOffA = kOffP + kMaxPRows * 256;
constexpr uint32_t kOffScale = kOffA + kStages * kStageBytes;                  // float [2][8][132]
constexpr uint32_t kOffLut = kOffScale + 2 * kMaxGroups * kScaleStride * 4;  // code LUT blob
constexpr uint32_t kOffFlags = kOffLut + (uint32_t)kCodeLutBytes;  // uint8 [2][4] zero-norm flags
constexpr uint32_t kOffMeta = kOffFlags + 16;
constexpr uint32_t kOffInfo = kOffMeta + ((sizeof(HeadMeta) + 15) & ~15);
constexpr uint32_t kOffBar = kOffInfo + 512;
constexpr int kNumBars = 18;
constexpr uint32_t kTcSmem = kOffBar + kNumBars * 8 + 16 + 1024;  // + slack for 1024-byte alignment
static_assert(kOffP % 1024 == 0 && kOffA % 1024 == 0, "swizzled operands need 1024-byte alignment");
static_assert(kTcSmem <= 232448, "shared memory budget");

// barrier indices
constexpr int kFull = 0;     // [3] X tile landed (TMA bytes)
constexpr int kEmpty = 3;    // [3] X stage free: both GEMMs done + 4 norm warps
constexpr int kPFull = 6;    // gather accumulator written
constexpr int kPEmpty = 7;   // gather accumulator read by the 4 norm warps
constexpr int kCFull = 8;    // [2] code accumulator written
constexpr int kCEmpty = 10;  // [2] code accumulator read by the 8 code warps
constexpr int kSFull = 12;   // [2] scales of a tile written by the 4 norm warps
constexpr int kSEmpty = 14;  // [2] scales read by the 8 code warps
constexpr int kRBar = 16;    // R image loaded
constexpr int kDrain = 17;   // after a failed wait: the MMAs issued so far are done

// per-CTA gather layout (built once)
struct GatherInfo {
  int n_rows;      // P rows (multiple of 16)
  int n_chunks;    // 8-row chunks that hold dims
  int n_groups;
  int pad;
  uint8_t chunk_group[kMaxChunks];
  uint8_t grp_row0[kMaxGroups];    // first P row of group g
  uint8_t grp_rows[kMaxGroups];    // dims of group g (= m)
  uint8_t grp_chunks[kMaxGroups];  // 8-row chunks of group g
  float sqrt_m[kMaxGroups];
  uint8_t row_dim[kMaxPRows];      // input dim of P row r (0xFF: padding)
};
static_assert(sizeof(GatherInfo) <= 512, "gather info");

__host__ __device__ constexpr uint32_t idesc_f16(int n) {
  // f32 accumulate, f16 A and B, both K-major, M = 128, N = n
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kMTile >> 4) << 24);
}

struct TcArgs {
  const uint8_t* bimg_k;  // per head, kBBytes each
  const uint8_t* bimg_v;  // one image
  const HeadMeta* meta;
  const float* thr;
  const uint8_t* code_lut;
  uint8_t* packed;
  int64_t n_tiles;        // packed tiles per head (capacity)
  int tile_bytes;
  int kb, vb, pairing, hkv;
  int64_t mt0, mt1;       // MMA tiles [mt0, mt1) of every head
  int ctas_k, ctas_v;     // CTAs per head of each role (blockIdx.x < ctas_k: keys)
  int* status;
  SeqMap sm;              // tile addresses and sequence lengths
  int64_t cap;            // t_capacity: lengths are clamped to it
};

__device__ __forceinline__ uint32_t su32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// bounded wait: gives up (returns false) after about two seconds.  Each try
// suspends the thread until the phase completes or a time hint expires, so a
// waiting warp takes no issue slots from the working ones.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  uint64_t t0 = 0;
  for (unsigned i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    if (ok) return true;
    if ((i & 15u) == 15u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0)
        t0 = now;
      else if (now - t0 > kTcWaitNs)
        return false;
    }
  }
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// shared-memory matrix descriptor: K-major, 128B swizzle, 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) |
         ((uint64_t)2 << 61);
}
__device__ __forceinline__ void tc_mma(uint32_t tmem, uint64_t da, uint64_t db, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
      "l"(da), "l"(db), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Per-lane constants of the code stage (the lane's coordinate has width w).
struct CodeLane {
  float inv, cadd;      // cell function of width w
  uint32_t lut_base;    // shared address of width w's entries minus 8 * bits(2^23)
  int lo, hi;           // clamp of the raw cell bits: bits(2^23) + [0, nmax]
  uint32_t sel_even, sel_odd;  // byte selectors of the merge with the partner lane
  uint32_t mA, mB, m2;  // byte pairs (1, 2^w) at bytes 0-1 / 2-3 and 2^(2w) for compressing
  uint32_t s4;          // 4w
  int w;
};

// Code of z: the number of thresholds t_i < z, from the cell table (one load,
// one comparison; exact because cells are monotone and hold one threshold).
__device__ __forceinline__ uint32_t code_of(float z, const CodeLane& L) {
  int b = __float_as_int(__fmaf_rz(z, L.inv, L.cadd));
  b = min(max(b, L.lo), L.hi);
  uint32_t tb, base;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(tb), "=r"(base) : "r"(L.lut_base + ((uint32_t)b << 3)));
  return base + (z > __uint_as_float(tb) ? 1u : 0u);
}

// Byte of the lane's code for token jj (0..63) of a packed tile: word jj_word,
// byte jj_byte of 16 words.  Keys: portion g = jj % 8 (8 codes u = jj / 8) in
// words 2g, 2g + 1.  Values: portion c = (jj / 2) % 4, own index 4b + 2k + l with
// jj = 16b + 8k + 2c + l, in words 4c + b.  Either way the lane with side s keeps
// words 8s..8s+7 (4 key portions g = 4s..4s+3 / 2 value portions c = 2s, 2s+1).
template <int ROLE>
__host__ __device__ constexpr int code_word(int jj) {
  return ROLE == 0 ? 2 * (jj & 7) + (jj >> 5) : 4 * ((jj >> 1) & 3) + (jj >> 4);
}
template <int ROLE>
__host__ __device__ constexpr int code_byte(int jj) {
  return ROLE == 0 ? (jj >> 3) & 3 : 2 * ((jj >> 3) & 1) + (jj & 1);
}

// Codes of 32 tokens (half HALF of the packed tile) into the lane's byte words.
template <int ROLE, int HALF, bool ZMASK>
__device__ __forceinline__ void code_half(const uint32_t (&y)[32], const float* sc,
                                          const CodeLane& L, uint32_t (&A)[16]) {
#pragma unroll
  for (int q4 = 0; q4 < 8; ++q4) {
    const float4 s4 = *reinterpret_cast<const float4*>(sc + 4 * q4);
    const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int jj = 32 * HALF + 4 * q4 + i;
      uint32_t code = code_of(__uint_as_float(y[4 * q4 + i]) * sv[i], L);
      if (ZMASK && sv[i] == 0.f) code = 0;  // zero vector (or zero group): codes 0
      A[code_word<ROLE>(jj)] |= code << (8 * code_byte<ROLE>(jj));
    }
  }
}

// Store 8 chunks of 8W bits (chunk k at bit 8W k): the lane's 8W bytes.
template <int W>
__device__ __forceinline__ void store_stream(const uint32_t (&clo)[8], const uint32_t (&chi)[8],
                                             uint8_t* dst) {
  uint32_t o[2 * W];
#pragma unroll
  for (int i = 0; i < 2 * W; ++i) o[i] = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int bit = 8 * W * k, w0 = bit >> 5, sh = bit & 31;
    if (sh == 0) {
      o[w0] |= clo[k];
      if (w0 + 1 < 2 * W) o[w0 + 1] |= chi[k];
    } else {
      o[w0] |= clo[k] << sh;
      if (w0 + 1 < 2 * W) o[w0 + 1] |= (clo[k] >> (32 - sh)) | (chi[k] << sh);
      if (w0 + 2 < 2 * W) o[w0 + 2] |= chi[k] >> (32 - sh);
    }
  }
#pragma unroll
  for (int i = 0; i < W; ++i)
    *reinterpret_cast<uint2*>(dst + 8 * i) = make_uint2(o[2 * i], o[2 * i + 1]);
}

// Merge with the partner lane, compress the 64 kept codes to W bits each and store.
__device__ __forceinline__ void pack_store(const uint32_t (&A)[16], const CodeLane& L,
                                           uint32_t side, int partner_xor, uint8_t* dst,
                                           bool store) {
  uint32_t keep[8], recv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t send = side ? A[i] : A[8 + i];
    keep[i] = side ? A[8 + i] : A[i];
    recv[i] = __shfl_xor_sync(0xffffffffu, send, partner_xor);
  }
  uint32_t clo[8], chi[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t v[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 2 * k + h;  // 4 consecutive codes of the stream, in stream order
      const uint32_t x = __byte_perm(keep[i >> 1], recv[i >> 1], (i & 1) ? L.sel_odd : L.sel_even);
      const uint32_t d0 = __dp4a(x, L.mA, 0u), d1 = __dp4a(x, L.mB, 0u);
      v[h] = L.w == 8 ? x : d0 + d1 * L.m2;
    }
    clo[k] = v[0] | __funnelshift_lc(0u, v[1], L.s4);
    chi[k] = __funnelshift_lc(v[1], 0u, L.s4);
  }
  if (!store) return;
  switch (L.w) {
    case 1: store_stream<1>(clo, chi, dst); break;
    case 2: store_stream<2>(clo, chi, dst); break;
    case 3: store_stream<3>(clo, chi, dst); break;
    case 4: store_stream<4>(clo, chi, dst); break;
    case 5: store_stream<5>(clo, chi, dst); break;
    case 6: store_stream<6>(clo, chi, dst); break;
    case 7: store_stream<7>(clo, chi, dst); break;
    case 8: store_stream<8>(clo, chi, dst); break;
    default: break;
  }
}

template <int ROLE>
__device__ __forceinline__ void tc_role(const CUtensorMap* tmap, const TcArgs& a, int cta,
                                        int n_cta) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = su32(sm);
  const int head = blockIdx.y, bidx = head / a.hkv, hidx = head % a.hkv;
  // tokens of this sequence: packed tiles starting at or past len are not written
  const int64_t len = a.sm.len(bidx, a.cap);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* scale = reinterpret_cast<float*>(sm + kOffScale);
  uint8_t* zflags = sm + kOffFlags;
  const CodeLutMeta* lut_meta = reinterpret_cast<const CodeLutMeta*>(sm + kOffLut);
  HeadMeta& m = *reinterpret_cast<HeadMeta*>(sm + kOffMeta);
  GatherInfo& gi = *reinterpret_cast<GatherInfo*>(sm + kOffInfo);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffBar + kNumBars * 8);
  const uint32_t bar0 = sb + kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(kFull + i), 1);
      mbar_init(bar(kEmpty + i), 1 + 4);
    }
    mbar_init(bar(kPFull), 1);
    mbar_init(bar(kPEmpty), 4);
    mbar_init(bar(kDrain), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kCFull + i), 1);
      mbar_init(bar(kCEmpty + i), 8);
      mbar_init(bar(kSFull + i), 4);
      mbar_init(bar(kSEmpty + i), 8);
    }
    mbar_init(bar(kRBar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < (int)(kCodeLutBytes / 16); i += kTcThreads)
    reinterpret_cast<uint4*>(sm + kOffLut)[i] = reinterpret_cast<const uint4*>(a.code_lut)[i];
  if (ROLE == 0) {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(a.meta + head);
    for (int i = tid; i < (int)(sizeof(HeadMeta) / 4); i += kTcThreads)
      reinterpret_cast<uint32_t*>(&m)[i] = src[i];
  }
  __syncthreads();
  if (tid == 0) {  // gather rows: the dims of every group in block order, groups padded to 8 rows
    int row = 0, ch = 0;
    const int ng = ROLE == 0 ? m.n_groups : 1;
    for (int g = 0; g < ng; ++g) {
      gi.grp_row0[g] = (uint8_t)row;
      int cnt = 0;
      if (ROLE == 0) {
        for (int b = 0; b < kBlocks; ++b)
          if (m.block_group[b] == g) {
            gi.row_dim[row + cnt++] = (uint8_t)(a.pairing == GTQ_PAIRING_HALF ? b : 2 * b);
            gi.row_dim[row + cnt++] = (uint8_t)(a.pairing == GTQ_PAIRING_HALF ? b + kBlocks : 2 * b + 1);
          }
        gi.sqrt_m[g] = m.sqrt_m[g];
      } else {
        for (int d = 0; d < kD; ++d) gi.row_dim[row + cnt++] = (uint8_t)d;
        gi.sqrt_m[g] = 11.313708498984761f;  // sqrt(128)
      }
      gi.grp_rows[g] = (uint8_t)cnt;
      const int nck = (cnt + 7) / 8;
      gi.grp_chunks[g] = (uint8_t)nck;
      for (int c = 0; c < nck; ++c) gi.chunk_group[ch + c] = (uint8_t)g;
      for (int r = cnt; r < 8 * nck; ++r) gi.row_dim[row + r] = 0xFF;
      row += 8 * nck;
      ch += nck;
    }
    gi.n_chunks = ch;
    gi.n_groups = ng;
    gi.n_rows = row < 16 ? 16 : (row + 15) & ~15;
    for (int r = row; r < gi.n_rows; ++r) gi.row_dim[r] = 0xFF;
  }
  __syncthreads();
  const int n_rows = gi.n_rows;
  if (ROLE == 0) {  // P image: zero, then one 1.0 per used row (keys only)
    uint4* p = reinterpret_cast<uint4*>(sm + kOffP);
    for (int i = tid; i < n_rows * 16; i += kTcThreads) p[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    for (int r = tid; r < n_rows; r += kTcThreads) {
      const int d = gi.row_dim[r];
      if (d != 0xFF)
        *reinterpret_cast<uint16_t*>(sm + kOffP + (d >> 6) * (n_rows * 128) + r * 128 +
                                     ((((d >> 3) & 7) ^ (r & 7)) << 4) + (d & 7) * 2) = 0x3C00;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
        su32(tmem_slot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int64_t n_mt = a.mt1 - a.mt0;
  int failed = 0, issued = 0;  // issued: tile copies the producer started
  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      const uint8_t* rsrc = ROLE == 0 ? a.bimg_k + (size_t)head * kBBytes : a.bimg_v;
      mbar_expect_tx(bar(kRBar), kBBytes);
      bulk_load(sb + kOffB, rsrc, kBBytes, bar(kRBar));
      int it = 0;
      for (int64_t t = cta; t < n_mt; t += n_cta, ++it) {
        const int st = it % kStages;
        if (!mbar_wait(bar(kEmpty + st), ((it / kStages) & 1) ^ 1)) { failed = 1; break; }
        issued = it + 1;
        const uint32_t dst = sb + kOffA + st * kStageBytes;
        const int row = (int)((a.mt0 + t) * kMTile);
        mbar_expect_tx(bar(kFull + st), kStageBytes);
        tma_load_4d(dst, tmap, 0, row, hidx, bidx, bar(kFull + st));
        tma_load_4d(dst + 16384, tmap, 64, row, hidx, bidx, bar(kFull + st));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      if (!mbar_wait(bar(kRBar), 0)) failed = 1;
      const uint32_t idc = idesc_f16(kD), idp = idesc_f16(n_rows);
      const uint32_t p_atom = (uint32_t)n_rows * 128;
      int it = 0;
      for (int64_t t = cta; t < n_mt && !failed; t += n_cta, ++it) {
        const int st = it % kStages, ac = it & 1;
        if (!mbar_wait(bar(kFull + st), (it / kStages) & 1)) { failed = 1; break; }
        const uint32_t x_base = sb + kOffA + st * kStageBytes;
        if (ROLE == 0) {  // gather: D_p = X . P^T (key groups' dims, exact)
          if (!mbar_wait(bar(kPEmpty), (it & 1) ^ 1)) { failed = 1; break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc_mma(tmem + 256, smem_desc(x_base + (ks >> 2) * 16384 + (ks & 3) * 32),
                   smem_desc(sb + kOffP + (ks >> 2) * p_atom + (ks & 3) * 32), idp, ks != 0);
          tc_commit(bar(kPFull));
        }
        if (!mbar_wait(bar(kCEmpty + ac), ((it >> 1) & 1) ^ 1)) { failed = 1; break; }
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // code: D_c = (R_hi + R_lo) . X^T
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
            tc_mma(tmem + (uint32_t)(ac * kD), smem_desc(sb + kOffB + part * 32768 + koff),
                   smem_desc(x_base + koff), idc, (part | ks) != 0);
          }
        }
        tc_commit(bar(kCFull + ac));
        tc_commit(bar(kEmpty + st));
      }
    }
  } else if (warp < 6) {
    // ----------------------------------------------------------- norm warps
    const int q = warp & 3, j = 32 * q + lane;  // token of the tile (= tensor-memory lane)
    const uint32_t trow = tmem + 256 + ((uint32_t)(32 * q) << 16);
    const int norm_off = ROLE == 0 ? key_norm_offset(a.kb, a.vb) : value_norm_offset(a.kb, a.vb);
    const int jj = j & 63, npos = 2 * ((jj & 7) * 8 + (jj >> 3));
    const int n_chunks = gi.n_chunks;
    int ovf = 0, it = 0;
    for (int64_t t = cta; t < n_mt; t += n_cta, ++it) {
      const int st = it % kStages, par = it & 1;
      if (ROLE == 0) {
        if (!mbar_wait(bar(kPFull), it & 1)) { failed = 1; break; }
      } else {
        if (!mbar_wait(bar(kFull + st), (it / kStages) & 1)) { failed = 1; break; }
      }
      if (!mbar_wait(bar(kSEmpty + par), ((it >> 1) & 1) ^ 1)) { failed = 1; break; }
      tc_fence_after();
      const int64_t tok = (a.mt0 + t) * 128 + j;
      const bool tile_ok = (tok & ~int64_t(63)) < len, tok_ok = tok < len;
      uint8_t* tile_base = tile_ok ? a.sm.tile(a.packed, head, (a.mt0 + t) * 2 + (j >> 6)) : nullptr;
      const uint8_t* xt = sm + kOffA + st * kStageBytes;
      float* sc_par = scale + par * kMaxGroups * kScaleStride;
      // Group sums of exact squares in fp32 (eight accumulators), and each group's
      // norm finished as soon as its sum is complete.  acc[i] held `terms` exact
      // squares: |n / ||x|| - 1| <= (terms + 2) / 2 + 1/2 units of 2^-24 (sum depth
      // terms - 1 + 3, halved by the root, plus its rounding); lo / hi add one each.
      // A group whose fp16 rounding that window leaves open is settled below.
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      unsigned ambm = 0, zm = 0;  // 2 bits per group: 1 fp16 rounding undecided, 2 overflow undecided
      uint32_t lh[kMaxGroups];    // fp16 candidates lo | hi << 16 of each group
      auto put = [&](int g) {
        const float S = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        const int terms = ROLE == 0 ? gi.grp_chunks[g] : 16;
        const float n = sqrtf(S);
        float r;
        asm("rsqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(S));
        const float delta = (0.5f * (float)terms + 4.f) * 5.9604645e-8f;
        const float lo = n * (1.f - delta), hi = n * (1.f + delta);
        const bool zero = S == 0.f, over = lo > 65504.f, strad = !over && hi > 65504.f;
        const uint16_t l16 = __half_as_ushort(__float2half_rn(fminf(lo, 65504.f)));
        const uint16_t h16 = __half_as_ushort(__float2half_rn(fminf(hi, 65504.f)));
        zm |= zero ? 1u : 0u;
        ovf |= (over && tok_ok) ? 1 : 0;
        ambm |= ((zero || over) ? 0u : (strad ? 2u : (l16 != h16 ? 1u : 0u))) << (2 * g);
        const uint32_t pk = (uint32_t)l16 | ((uint32_t)h16 << 16);
#pragma unroll
        for (int gg = 0; gg < kMaxGroups; ++gg)
          if (gg == g) lh[gg] = pk;
        if (tile_ok)
          *reinterpret_cast<uint16_t*>(tile_base + norm_off + g * 128 + npos) =
              zero ? (uint16_t)0 : (over ? (uint16_t)0x7BFF : l16);
        // scale of the codes (fp32, about 2^-22 relative)
        sc_par[g * kScaleStride + j] = zero ? 0.f : gi.sqrt_m[g] * r;
      };
      int ng;
      if (ROLE == 0) {
        // gathered exact inputs, 8 columns per chunk, 8 chunks per wait
        ng = gi.n_groups;
        int cur = 0;
        // a loop, not unrolled: this warp's code must stay small next to the code warps'
#pragma unroll 1
        for (int b = 0; b < n_chunks; b += 8) {
          uint32_t r0[32], r1[32];
          tc_ld32(trow + 8 * b, r0);
          tc_ld32(trow + 8 * b + 32, r1);
          tc_wait_ld();
          const uint2 cg = *reinterpret_cast<const uint2*>(&gi.chunk_group[b]);  // groups of chunks b..b+7
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (b + k < n_chunks) {
              const int g = (int)(((k < 4 ? cg.x : cg.y) >> (8 * (k & 3))) & 0xffu);
              if (g != cur) {
                put(cur);
                cur = g;
              }
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float x = __uint_as_float(k < 4 ? r0[8 * k + e] : r1[8 * (k - 4) + e]);
                acc[e] = fmaf(x, x, acc[e]);
              }
            }
          }
        }
        if (ng > 0) put(cur);
      } else {
        // values: one group of all 128 dims, straight from the fp16 tile (row j, 16-byte
        // chunk c at position c ^ (j % 8) of its 128-byte row)
        ng = 1;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(
              xt + (c >> 3) * 16384 + j * 128 + ((uint32_t)((c & 7) ^ (j & 7)) << 4));
          const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
          const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
          const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&v.z));
          const float2 f3 = __half22float2(*reinterpret_cast<const __half2*>(&v.w));
          acc[0] = fmaf(f0.x, f0.x, acc[0]); acc[1] = fmaf(f0.y, f0.y, acc[1]);
          acc[2] = fmaf(f1.x, f1.x, acc[2]); acc[3] = fmaf(f1.y, f1.y, acc[3]);
          acc[4] = fmaf(f2.x, f2.x, acc[4]); acc[5] = fmaf(f2.y, f2.y, acc[5]);
          acc[6] = fmaf(f3.x, f3.x, acc[6]); acc[7] = fmaf(f3.y, f3.y, acc[7]);
        }
        put(0);
      }
      const unsigned zero_any = __ballot_sync(0xffffffffu, zm != 0);
      if (__ballot_sync(0xffffffffu, ambm != 0)) {
#pragma unroll 1
        for (int g = 0; g < ng; ++g) {
          const unsigned amb_g = (ambm >> (2 * g)) & 3u;
          unsigned am = __ballot_sync(0xffffffffu, amb_g != 0);
          uint32_t pk = lh[0];
#pragma unroll
          for (int gg = 1; gg < kMaxGroups; ++gg)
            if (gg == g) pk = lh[gg];
          const uint16_t hlg = (uint16_t)(pk & 0xffffu), hhg = (uint16_t)(pk >> 16);
          while (am) {  // exact decision from the fp64 sum of squares, the whole warp helping
            const int src = __ffs(am) - 1;
            am &= am - 1;
            const int jt = 32 * q + src;
            double sq = 0.0;
            for (int rr = lane; rr < gi.grp_rows[g]; rr += 32) {
              const int d = gi.row_dim[gi.grp_row0[g] + rr];
              const __half x = *reinterpret_cast<const __half*>(
                  xt + (d >> 6) * 16384 + jt * 128 + ((((d >> 3) & 7) ^ (jt & 7)) << 4) + (d & 7) * 2);
              const double xd = (double)__half2float(x);
              sq = fma(xd, xd, sq);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
            if (lane == src) {
              uint16_t hb;
              if (amb_g == 1 && hhg == hlg + 1) {
                // n is between the two fp16 values: compare with their midpoint squared
                // (12 significant bits, exact in fp64); a tie rounds to even
                const double mid = 0.5 * ((double)__half2float(__ushort_as_half(hlg)) +
                                          (double)__half2float(__ushort_as_half(hhg)));
                const double m2 = mid * mid;
                hb = sq > m2 ? hhg : (sq < m2 ? hlg : ((hlg & 1) ? hhg : hlg));
              } else {
                const double n64 = sqrt(sq);
                if (n64 > 65504.0 && tok_ok) ovf = 1;
                hb = __half_as_ushort(__double2half(n64 > 65504.0 ? 65504.0 : n64));
              }
              if (tile_ok) *reinterpret_cast<uint16_t*>(tile_base + norm_off + g * 128 + npos) = hb;
            }
          }
        }
      }
      if (lane == 0) zflags[par * 4 + q] = zero_any ? 1 : 0;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (ROLE == 0) mbar_arrive(bar(kPEmpty));
        mbar_arrive(bar(kEmpty + st));
        mbar_arrive(bar(kSFull + par));
      }
    }
    if (ovf) atomicOr(a.status, kStatusOverflow);
  } else {
    // ----------------------------------------------------------- code warps
    const int q = warp & 3, hc = (warp - 6) >> 2;
    const int c = 32 * q + lane;  // rotated coordinate = tensor-memory lane
    int w, grp, dst_off;
    uint32_t side;
    if (ROLE == 0) {
      const int slot = c >> 1;
      w = slot < m.n_slots ? m.slot_width[slot] : 0;
      grp = slot < m.n_slots ? m.slot_group[slot] : 0;
      side = (uint32_t)(c & 1);
      dst_off = slot < m.n_slots ? m.slot_koff[slot] + 8 * w * (c & 1) : 0;
    } else {
      w = a.vb;
      grp = 0;
      side = (uint32_t)((c >> 3) & 1);
      dst_off = 1024 * a.kb + 16 * a.vb * (8 * (c >> 4) + (c & 7)) + 8 * a.vb * (int)side;
    }
    CodeLane L;
    {
      const int wl = w > 0 ? w : 1;  // width-0 lanes run width 1 and store nothing
      L.w = w;
      L.inv = lut_meta->inv[wl];
      L.cadd = lut_meta->cadd[wl];
      L.lut_base = sb + kOffLut + kCodeLutHeader + 8u * (uint32_t)lut_meta->off[wl] - 8u * 0x4B000000u;
      L.lo = 0x4B000000;
      L.hi = 0x4B000000 + lut_meta->nmax[wl];
      if (ROLE == 0) {  // stream quad = [E(u), O(u), E(u+1), O(u+1)], E = even coordinate
        L.sel_even = side ? 0x1504u : 0x5140u;
        L.sel_odd = side ? 0x3726u : 0x7362u;
      } else {          // stream quad = [E(l0), E(l1), O(l0), O(l1)], E = dim with h = 0
        L.sel_even = side ? 0x1054u : 0x5410u;
        L.sel_odd = side ? 0x3276u : 0x7632u;
      }
      const uint32_t p = 1u << wl;
      L.mA = 1u | ((p & 0xFFu) << 8);
      L.mB = (1u << 16) | ((p & 0xFFu) << 24);
      L.m2 = 1u << (2 * wl);
      L.s4 = 4u * (uint32_t)wl;
    }
    const int partner_xor = ROLE == 0 ? 1 : 8;
    const uint32_t tcol = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(64 * hc);
    int it = 0;
    for (int64_t t = cta; t < n_mt; t += n_cta, ++it) {
      const int ac = it & 1, par = it & 1;
      if (!mbar_wait(bar(kSFull + par), (it >> 1) & 1)) { failed = 1; break; }
      if (!mbar_wait(bar(kCFull + ac), (it >> 1) & 1)) { failed = 1; break; }
      tc_fence_after();
      const float* sc = scale + (par * kMaxGroups + grp) * kScaleStride + 64 * hc;
      const bool zmask = *reinterpret_cast<const uint32_t*>(zflags + par * 4) != 0;
      uint32_t A[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) A[i] = 0;
      {
        // both halves of the accumulator in one wait, then release it at once
        uint32_t y0[32], y1[32];
        tc_ld32(tcol + (uint32_t)(ac * kD), y0);
        tc_ld32(tcol + (uint32_t)(ac * kD) + 32, y1);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kCEmpty + ac));  // accumulator may be overwritten
        if (zmask) {
          code_half<ROLE, 0, true>(y0, sc, L, A);
          code_half<ROLE, 1, true>(y1, sc + 32, L, A);
        } else {
          code_half<ROLE, 0, false>(y0, sc, L, A);
          code_half<ROLE, 1, false>(y1, sc + 32, L, A);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kSEmpty + par));  // scales and flags read
      const int64_t ptile = (a.mt0 + t) * 2 + hc;
      const bool tile_ok = ptile * kTile < len;
      uint8_t* dst = tile_ok ? a.sm.tile(a.packed, head, ptile) + dst_off : nullptr;
      pack_store(A, L, side, partner_xor, dst, w > 0 && tile_ok);
    }
  }
  if (failed) atomicOr(a.status, kStatusTimeout);
  // After a failed wait, nothing in flight may outlive the CTA: the MMA issuer
  // waits (bounded) until its issued MMAs are done, the producer until every
  // tile copy it issued has landed.  Otherwise every copy and MMA was consumed.
  if (__syncthreads_or(failed)) {
    if (warp == 1 && lane == 0) {
      tc_commit(bar(kDrain));
      mbar_wait(bar(kDrain), 0);
    }
    if (warp == 0 && lane == 0)
      for (int st = 0; st < kStages && st < issued; ++st) {
        const int last = st + ((issued - 1 - st) / kStages) * kStages;  // last fill of the stage
        mbar_wait(bar(kFull + st), (last / kStages) & 1);
      }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

__global__ void __launch_bounds__(kTcThreads, 1)
    quantize_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, TcArgs a) {
  if ((int)blockIdx.x < a.ctas_k)
    tc_role<0>(&tmk, a, blockIdx.x, a.ctas_k);
  else
    tc_role<1>(&tmv, a, blockIdx.x - a.ctas_k, a.ctas_v);
}

// R image of a 128 x 128 matrix (rows = output coordinate, cols = input dim):
// fp16 hi part then fp16 lo part, each K-major with the 128B swizzle.
__global__ void b_image_kernel(const float* __restrict__ rows, size_t row_stride_heads,
                               uint8_t* __restrict__ img) {
  const float* r = rows + (size_t)blockIdx.x * row_stride_heads;
  uint8_t* o = img + (size_t)blockIdx.x * kBBytes;
  for (int i = threadIdx.x; i < kD * kD; i += blockDim.x) {
    const int n = i / kD, d = i % kD;
    const float v = r[i];
    const __half hi = __float2half_rn(v);
    const __half lo = __float2half_rn(v - __half2float(hi));
    const uint32_t off = (d >> 6) * 16384 + n * 128 + ((((d >> 3) & 7) ^ (n & 7)) << 4) + (d & 7) * 2;
    *reinterpret_cast<__half*>(o + off) = hi;
    *reinterpret_cast<__half*>(o + 32768 + off) = lo;
  }
}

// Raw cell bits of z in the code table: bits(fma(z, inv, cadd) rounded toward zero)
// minus bits(2^23) (the same expression the quantizer evaluates).
__device__ __forceinline__ int code_cell(float z, float inv, float cadd) {
  return __float_as_int(__fmaf_rz(z, inv, cadd)) - 0x4B000000;
}

// Builds the code table of widths 1..8 from the fp32 thresholds (one thread).
__global__ void code_lut_kernel(const float* __restrict__ thr, uint8_t* __restrict__ blob) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  CodeLutMeta* lm = reinterpret_cast<CodeLutMeta*>(blob);
  float2* cells = reinterpret_cast<float2*>(blob + kCodeLutHeader);
  for (int w = 0; w <= GTQ_MAX_BITS; ++w) {
    lm->inv[w] = 0.f;
    lm->cadd[w] = 8388608.f;
    lm->off[w] = 0;
    lm->nmax[w] = 0;
  }
  int off = 0, ok = 1;
  for (int w = 1; w <= GTQ_MAX_BITS && ok; ++w) {
    const float* t = thr + thr_base(w);
    const int nt = (1 << w) - 1;
    float gap = 1.f;
    for (int k = 1; k < nt; ++k) gap = fminf(gap, t[k] - t[k - 1]);
    const float inv = 1.f / (0.98f * gap);
    const int kofs = 2 - (int)floorf(t[0] * inv);  // the lowest threshold lands in cell >= 1
    const float cadd = 8388608.f + (float)kofs;
    const int n = code_cell(t[nt - 1], inv, cadd) + 2;  // the last cell holds no threshold
    if (code_cell(t[0], inv, cadd) < 1 || off + n > kCodeLutEntries) {
      ok = 0;
      break;
    }
    for (int i = 0; i < n; ++i) cells[off + i] = make_float2(INFINITY, __int_as_float(0));
    for (int k = 0; k < nt; ++k) {
      const int c = code_cell(t[k], inv, cadd);
      if (cells[off + c].x != INFINITY) ok = 0;
      cells[off + c].x = t[k];
    }
    int below = 0, k = 0;
    for (int i = 0; i < n; ++i) {
      while (k < nt && code_cell(t[k], inv, cadd) < i) {
        ++below;
        ++k;
      }
      cells[off + i].y = __int_as_float(below);
    }
    lm->inv[w] = inv;
    lm->cadd[w] = cadd;
    lm->off[w] = off;
    lm->nmax[w] = n - 1;
    off += n;
  }
  *reinterpret_cast<int*>(blob + kCodeLutOkOffset) = ok;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

bool encode_fp16_map(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box, bool swizzle128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = (cuuint64_t)dims[i];
    bx[i] = (cuuint32_t)box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = (cuuint64_t)strides[i];
  }
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (cuuint32_t)rank, const_cast<void*>(base), d, st,
             bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t build_b_images(const float* rows, int count, size_t stride, uint8_t* img,
                           cudaStream_t s) {
  b_image_kernel<<<count, 256, 0, s>>>(rows, stride, img);
  return cudaGetLastError();
}

size_t b_image_bytes() { return kBBytes; }

cudaError_t build_code_lut(const float* thr, uint8_t* blob, cudaStream_t s) {
  code_lut_kernel<<<1, 32, 0, s>>>(thr, blob);
  return cudaGetLastError();
}

// Quantize MMA tiles [mt0, mt1) of every head (keys and values in one launch).
// Returns cudaErrorNotSupported when the inputs cannot be described by a tensor map.
cudaError_t launch_quantize_tc(const gtq_plan* p, const void* k, const void* v, const int64_t* st,
                               int64_t mt0, int64_t mt1, uint8_t* packed, const SeqMap& sm,
                               cudaStream_t s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap maps[2];
  const void* src[2] = {k, v};
  if (p->cfg.v_bits == 0) src[1] = k;  // K-only: the value map is never used
  for (int r = 0; r < 2; ++r) {
    if (((uintptr_t)src[r] & 15) || ((st[0] * 2) & 15) || ((st[1] * 2) & 15) || ((st[2] * 2) & 15))
      return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)(mt1 * kMTile),
                                (cuuint64_t)p->cfg.n_kv_heads, (cuuint64_t)p->cfg.batch};
    const cuuint64_t strides[3] = {(cuuint64_t)st[2] * 2, (cuuint64_t)st[1] * 2,
                                   (cuuint64_t)st[0] * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)kMTile, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(&maps[r], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(src[r]), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  TcArgs a;
  a.bimg_k = p->d_bimg;
  a.bimg_v = p->tab.rv_image;
  a.meta = p->d_meta;
  a.thr = p->tab.thr;
  a.code_lut = p->tab.code_lut;
  a.packed = packed;
  a.n_tiles = p->n_tiles;
  a.tile_bytes = (int)p->tile_bytes;
  a.kb = p->cfg.k_bits;
  a.vb = p->cfg.v_bits;
  a.pairing = p->cfg.rope_pairing;
  a.hkv = p->cfg.n_kv_heads;
  a.mt0 = mt0;
  a.mt1 = mt1;
  a.status = p->d_status;
  a.sm = sm;
  a.cap = p->cfg.t_capacity;
  const int64_t n_mt = mt1 - mt0;
  // SMs per head are shared between the roles by their measured cost per tile
  // (a key tile costs about twice a value tile); every CTA keeps one head
  const int per_head = std::max(2, p->n_sms / std::max(1, p->n_heads));
  // The head's CTAs split between the roles (rounded share, at least one each),
  // key and value CTAs together within the head's share of the SMs.
  const bool konly = p->cfg.v_bits == 0;
  int share_k = std::min(per_head - 1, std::max(1, (per_head * kKeyShare + 50) / 100));
  int share_v = per_head - share_k;
  if (konly) {  // K-only: every CTA of the head codes keys
    share_k = per_head;
    share_v = 0;
  }
  if (per_head == 2) {
    // Many heads (fewer than three SMs each): each head takes 2u key CTAs and u
    // value CTAs (u key CTAs alone for K-only plans), since a key tile costs
    // about twice a value tile; the CTAs run in waves over the SMs.  u minimises
    // the estimated finish: waves x (the busiest CTA's tiles in value-tile units
    // + a set-up of about two value tiles).
    int best_u = 1;
    int64_t best = INT64_MAX;
    for (int u = 1; u <= 8; ++u) {
      const int ck = konly ? u : 2 * u, cv = konly ? 0 : u;
      const int64_t waves = ((int64_t)p->n_heads * (ck + cv) + p->n_sms - 1) / p->n_sms;
      const int64_t kt = (n_mt + ck - 1) / ck, vt = cv ? (n_mt + cv - 1) / cv : 0;
      const int64_t est = waves * (std::max(2 * kt, vt) + 2);
      if (est < best) {
        best = est;
        best_u = u;
      }
    }
    share_k = konly ? best_u : 2 * best_u;
    share_v = konly ? 0 : best_u;
  }
  a.ctas_k = (int)std::max<int64_t>(1, std::min<int64_t>(n_mt, share_k));
  a.ctas_v = konly ? 0 : (int)std::max<int64_t>(1, std::min<int64_t>(n_mt, share_v));
  cudaError_t e = cudaFuncSetAttribute(quantize_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmem);
  if (e != cudaSuccess) return e;
  quantize_tc_kernel<<<dim3(a.ctas_k + a.ctas_v, p->n_heads), kTcThreads, kTcSmem, s>>>(maps[0],
                                                                                        maps[1], a);
  return cudaGetLastError();
}

}  // namespace gtq
