// Internal declarations of libgtq (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gtq.h"

namespace gtq {

constexpr int kTile = GTQ_TILE_TOKENS;  // tokens per packed tile
constexpr int kD = 128;                 // head_dim of quantize / decode
constexpr int kBlocks = kD / 2;         // RoPE blocks per head
constexpr int kMaxGroups = 8;           // one group per nonzero width 1..8
constexpr int kMaxKt = 16;              // group-pure decode k-tiles: <= 8 + (groups - 1)
constexpr int kQSlice = 8;              // query heads one decode CTA serves (the MMA's N)
constexpr int kMaxGq = 128;             // query heads per KV head (decode: slices of kQSlice)
constexpr int kLutEntries = 510;        // sum over w = 1..8 of 2^w
constexpr int kThrEntries = 502;        // sum over w = 1..8 of (2^w - 1)
constexpr int kMaxSplits = 256;         // context splits per head in decode
constexpr int kPartialStride = 4 + kD;  // (m, l, -, -, o[128]) per (split, q head)
constexpr int kMergeGroup = 16;          // splits merged together at the first merge level
constexpr int kMaxMergeGroups = kMaxSplits / kMergeGroup;
constexpr int kWindowPartials = 16;     // fp16 window partials per head (at most)

// Context splits per head that a decode on n_heads heads may use (one CTA per
// SM; with many heads rounded up, so that late CTAs join heads with tiles left).
inline int decode_split_cap(int n_sms, int n_heads) {
  const int s = n_heads >= 16 ? (n_sms + n_heads - 1) / n_heads : (n_sms / n_heads > 1 ? n_sms / n_heads : 1);
  return s < kMaxSplits ? s : kMaxSplits;
}
// Partial slots of one decode unit: the splits, then the first-level group
// merges, then the window partials (one per split that attends window rows:
// at most kWindowPartials and at most the splits).
struct PartialSlots {
  int groups, window, total;
  explicit PartialSlots(int split_cap)
      : groups(split_cap),
        window(split_cap + (split_cap + kMergeGroup - 1) / kMergeGroup),
        total(window + (split_cap < kWindowPartials ? split_cap : kWindowPartials)) {}
};
constexpr int kMaxWindow = 1024;                // fp16 window rows per head (at most)
constexpr int kStatusOverflow = 1;      // status word bits
constexpr int kStatusTimeout = 2;
constexpr int kStatusLayout = 4;        // a kernel found its shared-memory layout unusable

// Byte offsets inside a packed tile: key codes, value codes (1024 vb), value
// norms (128, only when values are coded), key norms (128 per group).
__host__ __device__ constexpr int value_norm_offset(int kb, int vb) { return 1024 * (kb + vb); }
__host__ __device__ constexpr int key_norm_offset(int kb, int vb) {
  return 1024 * (kb + vb) + (vb > 0 ? 128 : 0);
}

// First LUT / threshold entry of width w (1..8).
__host__ __device__ inline int lut_base(int w) { return (1 << w) - 2; }
__host__ __device__ inline int thr_base(int w) { return (1 << w) - 1 - w; }

// Per-head metadata derived from the allocation (built on the device).
struct HeadMeta {
  int32_t n_groups;  // G_K: nonzero-width groups
  int32_t n_slots;   // sum over groups of m/2
  int32_t n_ktiles;  // decode k-tiles (16 coords each), every one inside one group
  int32_t reserved;
  float inv_sqrt_m[kMaxGroups];
  float sqrt_m[kMaxGroups];
  uint8_t grp_width[kMaxGroups];  // descending
  uint8_t grp_m[kMaxGroups];
  uint8_t grp_first_slot[kMaxGroups];
  uint8_t grp_split[kMaxGroups];  // decode computes this group's logits in split fp16
  uint8_t slot_width[kBlocks];
  uint8_t slot_group[kBlocks];
  uint16_t slot_koff[kBlocks];    // byte offset of the slot in the key-code area
  uint8_t block_group[kBlocks];   // group of each RoPE block (0xFF: width 0)
  uint8_t grp_kt0[kMaxGroups];    // decode k-tiles of group g: [grp_kt0, grp_kt1)
  uint8_t grp_kt1[kMaxGroups];
  uint8_t kt_group[kMaxKt];       // group of decode k-tile k
  uint8_t kt_first_slot[kMaxKt];  // its slots: [first, first + n)
  uint8_t kt_nslots[kMaxKt];      // 1..8
  uint8_t kt_flags[kMaxKt];       // bit 0: first k-tile of its group, bit 1: last
};

// Decode lookup tables, laid out exactly as the decode kernel's shared memory
// (one region whose shared address is a multiple of kDecTabAlign).  Every
// lookup address is "(region | index << 7 | lane bits) + table offset": the
// index is moved into place with one shift and merged with one mask-or, the
// table offset is the load's immediate.
//  * hi pair tables P32, widths 1..3: entry c0 | c1 << w is the fp16 half2
//    (cb[c0], cb[c1]) (hi parts), one copy per lane at entry * 128 + lane * 4:
//    a warp-wide 32-bit lookup never has a bank conflict;
//  * hi|lo pair tables P16, widths 1..4: entry c0 | c1 << w is the 8 bytes
//    {hi half2, lo half2} of (cb[c0], cb[c1]), one copy per lane pair at
//    entry * 128 + (lane & 15) * 8: a 64-bit lookup is two conflict-free
//    half-warp phases;
//  * hi|lo single-code tables S32, widths 5 and 6: entry c holds the fp16 hi
//    part (low half) and lo part (high half) of cb[c], at c * 128 + lane * 4;
//  * shared single-code table SS, widths 1..8 (same entry format), one copy at
//    kSingleOff(w) + c * 4 (widths 7 and 8, bank conflicts accepted).
// hi = fp16(cb), lo = fp16(cb - hi).
constexpr uint32_t kDecTabAlign = 32768;  // P16 width 4: 256 entries << 7
constexpr uint32_t kTabP16W4 = 0;
constexpr uint32_t kTabP16W3 = kTabP16W4 + (256u << 7);
constexpr uint32_t kTabP16W2 = kTabP16W3 + (64u << 7);
constexpr uint32_t kTabP16W1 = kTabP16W2 + (16u << 7);
constexpr uint32_t kTabP32W3 = kTabP16W1 + (4u << 7);
constexpr uint32_t kTabP32W2 = kTabP32W3 + (64u << 7);
constexpr uint32_t kTabP32W1 = kTabP32W2 + (16u << 7);
constexpr uint32_t kTabS32W5 = kTabP32W1 + (4u << 7);
constexpr uint32_t kTabS32W6 = kTabS32W5 + (32u << 7);
constexpr uint32_t kTabSS = kTabS32W6 + (64u << 7);
constexpr int kDecodeImageBytes = (int)(kTabSS + 2048u);
__host__ __device__ constexpr uint32_t kTabP16(int w) {
  return w == 4 ? kTabP16W4 : (w == 3 ? kTabP16W3 : (w == 2 ? kTabP16W2 : kTabP16W1));
}
__host__ __device__ constexpr uint32_t kTabP32(int w) {
  return w == 3 ? kTabP32W3 : (w == 2 ? kTabP32W2 : kTabP32W1);
}
__host__ __device__ constexpr uint32_t kTabS32(int w) { return w == 5 ? kTabS32W5 : kTabS32W6; }
__host__ __device__ constexpr uint32_t kSingleOff(int w) { return 2048u - (8u << w); }
static_assert(kDecodeImageBytes % 16 == 0 && kDecodeImageBytes <= 72 * 1024, "decode tables");

// Key rotation of one head for the decode kernel's query rotation
// ("rotation pack", fp32 words): words [0, 32) hold coord_dim[128] (uint8: the
// head dim of packed position p's group coordinate p - first(g)), then for
// every key group g in order its R_m transposed, m x m floats with element
// (c, r) = R_m[r][c] at word 32 + (sum over earlier groups of m^2) + c * m + r.
constexpr int kRotPackHeaderWords = 32;
constexpr int kRotPackMaxWords = kRotPackHeaderWords + kD * kD;
constexpr size_t kRotPackBytes = (size_t)kRotPackMaxWords * 4;

// Per-head split-merge counters of the decode kernel: [0] second-level
// ticket, [1, 1 + kMaxMergeGroups) first-level tickets, [kSchedWord] the
// dynamic tile counter.  Each is returned to 0 by the call that finishes with it.
constexpr int kSchedWord = 1 + kMaxMergeGroups;
constexpr int kTicketStride = kSchedWord + 1;

// Code lookup table of the tensor-core quantizer, one part per width w = 1..8.
// Cell of an fp32 value z: floor(z * inv[w]) + k[w], evaluated as
// fma(z, inv, 2^23 + k) rounded toward zero (the result's bits minus those of
// 2^23), clamped to [0, nmax].  The function is monotone, every cell holds at
// most one threshold T of width w (+inf if none), and the entry keeps T and the
// number of thresholds in lower cells, so the code #{t_i < z} = base + (z > T).
// Cell 0 and cell nmax hold no threshold.  Device blob: CodeLutMeta (kCodeLutHeader
// bytes) followed by float2 entries {T, base as int bits}.
constexpr int kCodeLutEntries = 1024;
struct CodeLutMeta {
  float inv[GTQ_MAX_BITS + 1];
  float cadd[GTQ_MAX_BITS + 1];  // 2^23 + k[w]
  int off[GTQ_MAX_BITS + 1];     // first entry of width w
  int nmax[GTQ_MAX_BITS + 1];    // last cell of width w
};
constexpr int kCodeLutHeader = 256;
static_assert(sizeof(CodeLutMeta) <= kCodeLutHeader - 4, "code LUT header");
constexpr int kCodeLutOkOffset = kCodeLutHeader - 4;  // int: 1 when the table is valid
constexpr size_t kCodeLutBytes = kCodeLutHeader + kCodeLutEntries * 8;

// Where the packed tile t of head (b, h) lives and how many tokens sequence b
// holds: contiguous per head (tile t of head at (head * n_tiles + t) tiles), or
// paged (block table row b: page table[b][t] holds tile t of every KV head of
// sequence b, head h at (page * hkv + h) tiles); lengths from seq_lens[b]
// (clamped to T) or T for all.
struct SeqMap {
  const int32_t* seq_lens = nullptr;
  const int32_t* table = nullptr;
  int64_t max_blocks = 0;
  int tail = 0;  // quantize: write the last n tokens of each sequence (t0 ignored)
  int hkv = 1;
  int64_t n_tiles = 0;
  int64_t tile_bytes = 0;
  __device__ __forceinline__ int64_t len(int b, int64_t T) const {
    if (!seq_lens) return T;
    const int64_t l = seq_lens[b];
    return l < 0 ? 0 : (l < T ? l : T);
  }
  __device__ __forceinline__ uint8_t* tile(uint8_t* packed, int head, int64_t t) const {
    if (table) {
      const int b = head / hkv, h = head % hkv;
      return packed + ((int64_t)table[(int64_t)b * max_blocks + t] * hkv + h) * tile_bytes;
    }
    return packed + ((int64_t)head * n_tiles + t) * tile_bytes;
  }
};

// Device-resident constant tables shared by every plan of a (device, seed).
struct Tables {
  double* rot_k;     // R_m for m = 2, 4, ..., 128, row-major, concatenated (fp64)
  float* rot_v;      // R_V 128 x 128 row-major (fp32)
  float* rot_vt;     // R_V^T (fp32): element [d][r] = R_V[r][d]
  uint32_t* rv_frag; // R_V^T as m16n8k16 A fragments, fp16 hi then lo (64 KB):
                     // word ((m * 8 + k) * 32 + lane) * 8 + {0..3 hi, 4..7 lo}
  double* dist;      // D(0..8)
  float* thr;        // fp32 thresholds, width w at thr_base(w)
  uint4* dec_image;  // kDecodeImageBytes: the decode kernel's lookup tables
  uint8_t* rv_image; // R_V as the quantizer's tensor-core B operand (fp16 hi + lo, 64 KB)
  uint8_t* code_lut; // kCodeLutBytes: CodeLutMeta + cells (built on the device from thr)
};

inline size_t rot_k_offset(int m) {  // element offset of R_m (m even) in rot_k
  size_t off = 0;
  for (int mm = 2; mm < m; mm += 2) off += (size_t)mm * mm;
  return off;
}
inline size_t rot_k_total() { return rot_k_offset(kD + 2); }

}  // namespace gtq

// Opaque plan (C ABI type).
struct gtq_plan {
  gtq_config cfg;
  int device;
  int n_heads;        // batch * n_kv_heads
  int n_blocks;       // head_dim / 2
  int g_q;            // n_q_heads / n_kv_heads
  int n_qs;           // query slices per KV head: ceil(g_q / kQSlice)
  int n_units;        // decode units: n_heads * n_qs (KV head, query slice) pairs
  int64_t n_tiles;    // tiles per head (capacity)
  size_t tile_bytes;
  size_t packed_bytes;
  int n_sms;
  gtq::Tables tab;    // borrowed from the library cache (not freed by the plan)
  double* d_energy;   // [heads][n_blocks]
  uint8_t* d_bits;    // [heads][n_blocks]
  gtq::HeadMeta* d_meta;  // [heads]
  float* d_mrow;      // [heads][128][128] key rotation rows in packed order (fp32)
  float* d_rotpack;   // [heads][kRotPackMaxWords] key rotation blocks for the decode kernel
  uint8_t* d_bimg;    // [heads] M_h as the quantizer's tensor-core B operand (64 KB each)
  float* d_partials;  // [units][PartialSlots(decode_split_cap).total][8][kPartialStride]
  unsigned* d_tickets;  // [units][kTicketStride] split-merge tickets and the tile counter
  int* d_status;      // device status word
};

namespace gtq {
// Error text for gtq_last_error (gtq_api.cu)
void set_last_error(const char* msg);
int record_cuda_error(cudaError_t e);  // GTQ_OK, or GTQ_ERR_CUDA / GTQ_ERR_OOM with the text set

// Host tables (gtq_tables.cu)
int lloyd_max_host(int bits, double* c, double* t, double* d);
int rotation_host(uint64_t seed, int tag, int m, double* out);
int tables_for(int device, uint64_t seed, Tables* out);  // cached per (device, seed)

// Kernel launchers
cudaError_t launch_energy(const gtq_plan* p, const void* k, int64_t T, const int64_t* st,
                          const int32_t* seq_lens, cudaStream_t s);
SeqMap seq_map(const gtq_plan* p, const gtq_seq_layout* lay);
cudaError_t launch_greedy_and_meta(const gtq_plan* p, cudaStream_t s);
cudaError_t launch_quantize(const gtq_plan* p, const void* k, const void* v, const int64_t* st,
                            int64_t t0, int64_t n, uint8_t* packed, const SeqMap& sm,
                            cudaStream_t s);
cudaError_t launch_quantize_cc(const gtq_plan* p, const void* k, const void* v, const int64_t* st,
                               int64_t t0, int64_t n, uint8_t* packed, const SeqMap& sm,
                               cudaStream_t s);
constexpr int kAppendMax = 16;  // tokens per call handled by the append kernel
cudaError_t launch_append(const gtq_plan* p, const void* k, const void* v, const int64_t* st,
                          int64_t t0, int64_t n, uint8_t* packed, const SeqMap& sm, cudaStream_t s);
cudaError_t launch_quantize_tc(const gtq_plan* p, const void* k, const void* v, const int64_t* st,
                               int64_t mt0, int64_t mt1, uint8_t* packed, const SeqMap& sm,
                               cudaStream_t s);
cudaError_t build_b_images(const float* rows, int count, size_t stride, uint8_t* img,
                           cudaStream_t s);
size_t b_image_bytes();
cudaError_t build_code_lut(const float* thr, uint8_t* blob, cudaStream_t s);
// Encodes a tiled fp16 tensor map (zero fill outside the extents); false if the
// driver entry point is missing or rejects the description.  strides: bytes of
// dims 1..rank-1.
bool encode_fp16_map(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box, bool swizzle128);

// fp16 operands of a decode (gtq_fp16_kv, checked): values of a K-only plan
// and the window of recent tokens; strides in elements
struct Fp16Kv {
  const __half* v = nullptr;
  int64_t vs[4] = {0, 0, 0, 0};
  const __half* rk = nullptr;
  const __half* rv = nullptr;
  int64_t rs[4] = {0, 0, 0, 0};
  const int32_t* rlens = nullptr;
  int64_t rlen = 0;
};
cudaError_t launch_decode(const gtq_plan* p, const uint8_t* packed, int64_t T, const void* q,
                          int q_dtype, float* out, const SeqMap& sm, const Fp16Kv& kv,
                          cudaStream_t s);
}  // namespace gtq
