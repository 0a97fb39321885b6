/*
 * gtq.h -- C ABI of libgtq: Block-GTQ packed KV cache on NVIDIA B200 (sm_100a).
 *
 * Block-GTQ ("RoPE-Aware Bit Allocation for KV-Cache Quantization", Liang,
 * Zhang, Jia; arXiv 2606.24033, Abstract) quantizes a key cache with
 * TurboQuant-MSE as the base quantizer: for each layer and KV head it scores
 * every 2-D RoPE block with an energy that needs no labels and gives out
 * integer bit widths one bit at a time by marginal gain; decoding then reads
 * the packed cache directly.  This library implements that hot path:
 *
 *   gtq_alloc_bits     energy of each RoPE block + greedy bit allocation
 *   gtq_quantize_pack  TQ-MSE group coding of K (mixed widths) and V (uniform)
 *                      into the packed cache
 *   gtq_decode_attn    fused GQA decode attention read directly from the codes
 *   gtq_free           release a plan
 *
 * Construction (the page gives the ideas, not formulas; these are the readings
 * this library implements):
 *   - RoPE blocks: HALF pairs dims (i, i + d/2), INTERLEAVED pairs (2i, 2i+1).
 *   - Energy E_i = (1/T) sum_t (k_t[p0]^2 + k_t[p1]^2) over the post-RoPE keys of
 *     one (sequence, KV head) of one layer, in fp64.
 *   - Greedy: from b_i = 0, repeatedly add one bit to the block with the largest
 *     E_i (D(b_i) - D(b_i + 1)) (D = Lloyd-Max MSE of N(0,1); ties to the lower
 *     index; widths capped at max_bits = 8) until sum_i 2 b_i = k_bits * d.
 *   - Groups: blocks of equal nonzero width w form one group of m = 2 * count
 *     coordinates (blocks ascending, p0 then p1).  Per token the group stores
 *     fp16(||k_g||) and the w-bit Lloyd-Max codes of sqrt(m) R_m k_g / ||k_g||,
 *     R_m a fixed seeded m x m orthogonal matrix (QR of a SplitMix64/Box-Muller
 *     Gaussian, diag(R) > 0).  Values: one group of all 128 dims, v_bits each,
 *     matrix R_V.  Zero vectors store norm 0 and codes 0.
 *   - Decode: s_t = (1/sqrt(d)) sum_g fp16(n_tg)/sqrt(m_g) (R_g q_g).cb[c_tg];
 *     online softmax over the T cached tokens; o = R_V^T sum_t p_t
 *     fp16(n_Vt)/sqrt(d) cb[c_Vt].  No fp16 K or V is ever materialised.
 *
 * Conventions for every entry point
 *   - Pointers named *_dev are CUDA device pointers owned by the caller; the
 *     library never frees or retains them past the call.  Host pointers are
 *     read or written before the call returns unless stated otherwise.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued asynchronously; no entry point synchronises the host
 *     except gtq_get_bits and gtq_status.
 *   - Return value: GTQ_OK (0) or a negative GTQ_ERR_* code.  On any error no
 *     work is enqueued and outputs are untouched.  gtq_strerror names a code.
 *   - A plan (gtq_plan) is one layer: batch x n_kv_heads independent heads.  It
 *     is owned by the library (created by gtq_alloc_bits*, released by gtq_free)
 *     and holds the allocation, per-head metadata, rotations, codebooks and
 *     decode workspace.  Calls on one plan must be ordered (same stream or
 *     explicit dependencies); plans are independent of one another.
 *   - Device-side faults of the data (a norm above the fp16 range, a bounded
 *     wait that expired) set a status word read by gtq_status; kernels never
 *     trap.
 */
#ifndef GTQ_H
#define GTQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GTQ_API __attribute__((visibility("default")))
#else
#define GTQ_API
#endif

#define GTQ_OK 0
#define GTQ_ERR_INVALID (-1)     /* bad argument: null, size, alignment, range   */
#define GTQ_ERR_UNSUPPORTED (-2) /* valid but not implemented (e.g. head_dim)     */
#define GTQ_ERR_CUDA (-3)        /* a CUDA runtime call failed                    */
#define GTQ_ERR_OOM (-4)         /* device allocation failed                      */
#define GTQ_ERR_TIMEOUT (-5)     /* a bounded device wait expired (status word)   */
#define GTQ_ERR_OVERFLOW (-6)    /* a norm exceeded 65504 and was clamped         */
#define GTQ_ERR_STATE (-7)       /* plan not ready for this call                  */

#define GTQ_PAIRING_HALF 0        /* RoPE block i = dims (i, i + d/2)  */
#define GTQ_PAIRING_INTERLEAVED 1 /* RoPE block i = dims (2i, 2i + 1)  */

#define GTQ_DTYPE_FP16 0
#define GTQ_DTYPE_FP32 1

#define GTQ_TILE_TOKENS 64 /* tokens per packed tile */
#define GTQ_MAX_BITS 8     /* widest code of any block */

typedef struct gtq_plan gtq_plan; /* opaque, library-owned */

/* One layer's configuration.  Sizes in elements. */
typedef struct gtq_config {
  int32_t batch;        /* sequences B >= 1; B * n_kv_heads <= 65535            */
  int32_t n_q_heads;    /* Hq, a multiple of n_kv_heads                         */
  int32_t n_kv_heads;   /* Hkv >= 1; Hq / Hkv (the GQA group) must be 1..128    */
  int32_t head_dim;     /* d: 128 for quantize/decode; any even 4..128 for alloc*/
  int32_t k_bits;       /* key budget in bits per dim, 1..8                     */
  int32_t v_bits;       /* value bits per dim, 1..8; 0: K-only (fp16 values)    */
  int32_t max_bits;     /* widest block width, 1..8 (normally 8)                */
  int32_t rope_pairing; /* GTQ_PAIRING_*                                        */
  int32_t in_dtype;     /* GTQ_DTYPE_* of K and V                               */
  int32_t reserved;     /* must be 0                                            */
  uint64_t seed;        /* rotation seed (R_m and R_V); 0 by default            */
  int64_t t_capacity;   /* tokens the packed cache holds per head (>= 1)        */
} gtq_config;

/*
 * gtq_alloc_bits -- energy pass + greedy allocation (the page's per-block
 * energy score and its one-bit-at-a-time marginal-gain allocation, Abstract).
 *   cfg        configuration (copied).
 *   k_dev      post-RoPE keys, in_dtype, element (b, h, t, i) at
 *              k_dev + b*k_strides[0] + h*k_strides[1] + t*k_strides[2] + i*k_strides[3]
 *              (strides in elements; k_strides[3] must be 1; rows 16-byte aligned).
 *   T          tokens to score, 1 <= T <= cfg->t_capacity.
 *   k_strides  4 element strides (host array).
 *   stream     cudaStream_t.
 *   out        receives the new plan (set only on success).
 * Creates the plan, allocates its device memory (cudaMalloc; this call is not
 * capturable), and enqueues the energy, greedy and per-head metadata kernels.
 * Errors: INVALID (null, bad sizes/strides/alignment, bits out of range, Hq not
 * a multiple of Hkv), UNSUPPORTED (group > 128, batch * Hkv > 65535, head_dim not
 * even 4..128), OOM, CUDA.
 */
GTQ_API int gtq_alloc_bits(const gtq_config* cfg, const void* k_dev, int64_t T,
                   const int64_t k_strides[4], void* stream, gtq_plan** out);

/*
 * gtq_alloc_bits_from_energy -- same plan, but the per-block energies are given
 * (host fp64 array [batch][n_kv_heads][head_dim/2]) instead of computed from K.
 * The greedy allocation and metadata still run on the device (enqueued on the
 * legacy default stream, synchronised before return).  Used to test the
 * allocator on chosen energies.  Errors as gtq_alloc_bits.
 */
GTQ_API int gtq_alloc_bits_from_energy(const gtq_config* cfg, const double* host_energy,
                               gtq_plan** out);

/*
 * gtq_quantize_pack -- TQ-MSE coding of keys (Block-GTQ mixed widths) and values
 * (uniform v_bits) of tokens [t0, t0 + n_tokens) into the packed cache.
 *   k_dev, v_dev  post-RoPE K and V, in_dtype, laid out like gtq_alloc_bits'
 *                 k_dev with the same 4 strides (strides[3] == 1); token t of
 *                 the cache is row t of these tensors.  A K-only plan
 *                 (v_bits 0) codes keys alone and takes v_dev = NULL.
 *   packed_dev    the packed cache, >= gtq_packed_bytes(plan) bytes, 16-byte
 *                 aligned, caller-owned.  Tokens outside [t0, t0+n) keep their
 *                 bytes (appending to an existing cache is allowed).
 *   packed_bytes  size of packed_dev in bytes.
 * Requires head_dim == 128 and t0 + n_tokens <= t_capacity.  A norm above 65504
 * is stored as 65504 and sets GTQ_ERR_OVERFLOW in the status word.  fp32 input
 * outside the fp16 range is not supported (its codes are undefined).
 * Errors: INVALID, UNSUPPORTED, CUDA.
 */
GTQ_API int gtq_quantize_pack(gtq_plan* plan, const void* k_dev, const void* v_dev,
                      const int64_t strides[4], int64_t t0, int64_t n_tokens,
                      void* packed_dev, size_t packed_bytes, void* stream);

/*
 * gtq_decode_attn -- fused GQA decode attention of one query token per sequence
 * over the first T tokens of the packed cache (the page decodes straight from
 * the packed cache, Abstract).  Scores are taken in each group's rotated basis, softmax is online and
 * split over the context, P.V accumulates in V's rotated basis and R_V^T is
 * applied once when the splits merge.
 *   packed_dev  cache written by gtq_quantize_pack for tokens [0, T).
 *   T           1 <= T <= t_capacity.
 *   q_dev       post-RoPE queries [batch][n_q_heads][128], q_dtype, contiguous,
 *               16-byte aligned.  Query head hq uses KV head hq / (Hq / Hkv).
 *   out_dev     fp32 [batch][n_q_heads][128], contiguous, 16-byte aligned, written
 *               in full.
 * Uses the plan's workspace: concurrent decodes on one plan must not overlap.
 * Errors: INVALID, UNSUPPORTED (head_dim != 128), STATE, CUDA.
 */
GTQ_API int gtq_decode_attn(gtq_plan* plan, const void* packed_dev, int64_t T,
                    const void* q_dev, int32_t q_dtype, float* out_dev, void* stream);
/* (A K-only plan, v_bits 0, decodes through gtq_decode_attn_full below.) */

/* ---- batches of sequences of their own lengths; paged caches ------------ */

/*
 * How the sequences of a batch are laid out (the page's serving setting of
 * Abstract, with requests of different lengths; a layout of this library's own).
 *   seq_lens_dev     device int32 [batch]: tokens held by sequence b (values
 *                    above the call's T are clamped to T, below 0 to 0), or
 *                    NULL: every sequence holds the call's T tokens.
 *   block_table_dev  device int32 [batch][max_blocks], or NULL: the packed
 *                    cache is contiguous, as gtq_packed_bytes describes.  With a
 *                    table, the packed buffer is a pool of pages; a page holds
 *                    one 64-token tile of every KV head of one sequence, and
 *                    tile n of head (b, h) sits at byte offset
 *                        ((block_table[b][n] * n_kv_heads + h) * tile_bytes)
 *                    of the pool (tile_bytes = gtq_layout_tile_bytes).  Every
 *                    entry a call touches (tiles below ceil(len_b / 64)) must
 *                    name a page inside the pool; the library does not read
 *                    the table on the host and cannot check it.
 *   max_blocks       columns of the block table (>= 1 with a table).
 * Both arrays are read by the kernels, on the call's stream, in stream order.
 */
typedef struct gtq_seq_layout {
  const int32_t* seq_lens_dev;
  const int32_t* block_table_dev;
  int64_t max_blocks;
} gtq_seq_layout;

/* gtq_alloc_bits with per-sequence lengths: E_i of sequence b is the mean over
 * its own first len_b tokens (0 for an empty sequence, whose greedy then gives
 * every bit to the lowest eligible block: ties go to the lower index).  lay may
 * be NULL.  Errors as gtq_alloc_bits. */
GTQ_API int gtq_alloc_bits_ex(const gtq_config* cfg, const void* k_dev, int64_t T,
                              const int64_t k_strides[4], const gtq_seq_layout* lay,
                              void* stream, gtq_plan** out);

/* gtq_quantize_pack into a layout: tokens [t0, t0 + n_tokens) of sequence b
 * are written only below len_b; with a block table the tiles go to the pool's
 * pages (packed_bytes = the pool's size, checked only against one page).
 * t0 = GTQ_T0_TAIL writes the last n_tokens tokens of every sequence instead,
 * [max(0, len_b - n_tokens), len_b) -- a batched decode-time append where each
 * sequence has grown to its own length (needs seq_lens_dev).  lay may be NULL
 * otherwise.  Errors as gtq_quantize_pack. */
#define GTQ_T0_TAIL (-1)
GTQ_API int gtq_quantize_pack_ex(gtq_plan* plan, const void* k_dev, const void* v_dev,
                                 const int64_t strides[4], int64_t t0, int64_t n_tokens,
                                 void* packed_dev, size_t packed_bytes,
                                 const gtq_seq_layout* lay, void* stream);

/* gtq_decode_attn over a layout: sequence b attends to its first len_b tokens
 * (T is an upper bound, <= t_capacity, that sizes the launch; a sequence of
 * length 0 gets a zero output).  lay may be NULL.  Errors as gtq_decode_attn;
 * a K-only plan needs gtq_decode_attn_full (INVALID here). */
GTQ_API int gtq_decode_attn_ex(gtq_plan* plan, const void* packed_dev, int64_t T,
                               const gtq_seq_layout* lay, const void* q_dev, int32_t q_dtype,
                               float* out_dev, void* stream);

/*
 * fp16 operands of a decode.
 *
 * K-only mode: a plan made with v_bits = 0 codes only the keys (the page's
 * K-only quantization, Abstract); the values stay in fp16 in the caller's own
 * cache and v_dev names them:
 *   v_dev           fp16, element (b, h, t, i) at v_dev + b*v_strides[0] +
 *                   h*v_strides[1] + t*v_strides[2] + i (v_strides[3] must be
 *                   1; the others multiples of 8; v_dev 16-byte aligned).
 *                   Rows t < the call's T are read (row t of sequence b only
 *                   below len_b, as the keys), whatever layout the packed keys
 *                   use.  NULL for plans with coded values.
 * Recent window: the fp16 recent-key buffer the page's headline result does
 * without (Abstract) -- the last tokens of a sequence kept in fp16 beside the
 * packed cache.  The query attends to the packed tokens and the window rows in
 * one softmax; window logits are q.k / sqrt(d) on the fp16 keys, window
 * values the fp16 values (original basis).
 *   recent_k_dev, recent_v_dev  fp16 post-RoPE keys and values, element
 *                   (b, h, r, i) at base + b*recent_strides[0] +
 *                   h*recent_strides[1] + r*recent_strides[2] + i
 *                   (recent_strides[3] must be 1, the others multiples of 8;
 *                   bases 16-byte aligned).
 *   recent_lens_dev device int32 [batch]: window rows of sequence b (clamped
 *                   to [0, recent_len]), or NULL: recent_len for every one.
 *   recent_len      rows per head, 0..1024; 0 = no window (the pointers may
 *                   then be NULL).
 * The window is attended on the tensor cores in blocks of 32 rows spread over
 * up to 16 CTAs of each KV head, each of which writes a partial of its own.
 */
typedef struct gtq_fp16_kv {
  const void* v_dev;
  int64_t v_strides[4];
  const void* recent_k_dev;
  const void* recent_v_dev;
  int64_t recent_strides[4];
  const int32_t* recent_lens_dev;
  int64_t recent_len;
} gtq_fp16_kv;

/* gtq_decode_attn_ex with fp16 operands (kv may be NULL: none).  A K-only plan
 * requires kv->v_dev, a plan with coded values forbids it.  A sequence whose
 * packed part and window are both empty gets a zero output.
 * Errors as gtq_decode_attn; INVALID also for a bad kv. */
GTQ_API int gtq_decode_attn_full(gtq_plan* plan, const void* packed_dev, int64_t T,
                                 const gtq_seq_layout* lay, const gtq_fp16_kv* kv,
                                 const void* q_dev, int32_t q_dtype, float* out_dev,
                                 void* stream);

/* gtq_free -- release the plan and its device memory.  Synchronises the plan's
 * device (cudaFree).  NULL is accepted.  Returns GTQ_OK or GTQ_ERR_CUDA. */
GTQ_API int gtq_free(gtq_plan* plan);

/* ---- helpers the page does not name (this library's additions) ---------- */

/* Bytes of the packed cache for cfg->t_capacity tokens of every head (0 on a
 * NULL plan).  Layout: see gtq_layout_* below. */
GTQ_API size_t gtq_packed_bytes(const gtq_plan* plan);

/* Copy the allocation to the host: bits[batch][n_kv_heads][head_dim/2] (uint8).
 * Synchronises `stream`.  Errors: INVALID, CUDA. */
GTQ_API int gtq_get_bits(gtq_plan* plan, uint8_t* host_bits, void* stream);

/* Copy the energies to the host: fp64 [batch][n_kv_heads][head_dim/2].
 * Synchronises `stream`.  Errors: INVALID, CUDA. */
GTQ_API int gtq_get_energy(gtq_plan* plan, double* host_energy, void* stream);

/* Read and clear the plan's device status word (synchronises the device):
 * GTQ_OK, GTQ_ERR_OVERFLOW or GTQ_ERR_TIMEOUT.  After GTQ_ERR_TIMEOUT the
 * outputs of the calls since the last check are undefined and so is the
 * plan's split-merge state: free the plan and build a new one. */
GTQ_API int gtq_status(gtq_plan* plan);

/* Device memory owned by the plan, in bytes (0 on NULL): energies, widths,
 * metadata, rotation rows and images, split-merge partials and counters; the
 * per-device constant tables and the caller's buffers are not counted. */
GTQ_API size_t gtq_plan_device_bytes(const gtq_plan* plan);

/*
 * gtq_raise_status -- set a condition in the plan's device status word from
 * the host, exactly as a kernel does when it meets it (code GTQ_ERR_TIMEOUT:
 * a bounded wait expired; GTQ_ERR_OVERFLOW: a norm was clamped).  It lets a
 * caller test its handling of gtq_status without making a GPU fault or hang.
 * Synchronises the device.  Errors: INVALID (NULL plan or another code), CUDA.
 */
GTQ_API int gtq_raise_status(gtq_plan* plan, int32_t code);

/* Human-readable name of a return code (static string). */
GTQ_API const char* gtq_strerror(int code);

/* Name and text of the last CUDA error an entry point of this thread turned
 * into GTQ_ERR_CUDA / GTQ_ERR_OOM ("" if none); valid until the next call. */
GTQ_API const char* gtq_last_error(void);

/*
 * gtq_block_energy_noalloc -- the energy pass of gtq_alloc_bits (E_i of every
 * RoPE block of every (sequence, KV head), fp64, same kernels and summation
 * order) without allocating any device memory.  The page has no counterpart:
 * this entry point serves callers that cannot call cudaMalloc at call time --
 * code running while a CUDA graph is captured, servers that reserve all
 * device memory up front, real-time loops that cannot afford the allocator.
 *   cfg         batch, n_kv_heads, head_dim (multiple of 8, <= 128),
 *               rope_pairing and in_dtype are read; other fields are ignored.
 *   k_dev       post-RoPE keys as in gtq_alloc_bits (same strides and alignment).
 *   T           tokens to score, >= 1.
 *   energy_dev  output, fp64 [batch][n_kv_heads][head_dim/2], 8-byte aligned,
 *               caller-owned device memory, written in full.
 * Scratch: a fixed 4 MiB array of partial sums inside the library (one per GPU
 * that loads it, held until the process exits).  batch * n_kv_heads *
 * ceil(T / 1024) * 128 must not exceed 2^19; larger calls return
 * GTQ_ERR_UNSUPPORTED (gtq_last_error gives the sizes) and launch nothing.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * All calls share the array: calls that overlap on the GPU (different streams
 * without ordering) race and give wrong energies.  Every scratch element a call
 * reads it has written first, so no clearing is needed between calls.
 * Errors: INVALID, UNSUPPORTED, CUDA.
 */
GTQ_API int gtq_block_energy_noalloc(const gtq_config* cfg, const void* k_dev, int64_t T,
                                     const int64_t k_strides[4], double* energy_dev,
                                     void* stream);

/* Library's own tables, computed on the host (no GPU needed):
 * the b-bit Lloyd-Max quantizer of N(0,1) (b = 0..8): 2^b centroids
 * (ascending), 2^b - 1 thresholds and the distortion D(b). */
GTQ_API int gtq_lloyd_max(int32_t bits, double* centroids, double* thresholds, double* distortion);

/* The seeded m x m rotation (row-major, fp64): tag 'K' (0x4B) for key groups of
 * size m (even, 2..128), tag 'V' (0x56) with m = 128 for values. */
GTQ_API int gtq_rotation(uint64_t seed, int32_t tag, int32_t m, double* out);

/*
 * Packed-cache layout (version 1).  Per head (b, h) the cache is
 * ceil(t_capacity / 64) tiles of gtq_layout_tile_bytes(k_bits, v_bits) bytes,
 * head-major: tile n of head (b, h) starts at
 *     ((b * n_kv_heads + h) * n_tiles + n) * tile_bytes.
 * Inside a tile (64 tokens; token j of the tile is t = 64 n + j):
 *   [0, 1024 k_bits)           key codes, by "slot".  The nonzero-width groups
 *                              are listed in DESCENDING width; the m rows of a
 *                              group's rotated vector (row r of R_m) form m/2
 *                              slots (rows 2s', 2s'+1).  Slot s of width w is
 *                              16 w bytes; within it, 8 portions g = 0..7 of
 *                              2 w bytes hold tokens j = g + 8 u (u = 0..7):
 *                              code (u, e) (e = row parity) at bits
 *                              [(2u+e) w, (2u+e+1) w), little-endian bit order.
 *   [1024 k_bits, +1024 v_bits) value codes: 256 portions p = (i*8 + g)*4 + c of
 *                              4 v_bits bytes (i = 0..7 dim tile, g, c = 0..3);
 *                              code x (x = 0..31) of portion p is dim
 *                              16 i + g + 8 (x>>1 & 1), token
 *                              16 (x>>3) + 2c + (x & 1) + 8 (x>>2 & 1), at bits
 *                              [x v_bits, (x+1) v_bits).  Dim = row of R_V.
 *   next 128 bytes             value norms, fp16 [g][u] -> token g + 8u
 *                              (absent, like the value codes, when v_bits = 0).
 *   next 128 * 8 bytes         key norms, fp16 [group][g][u] (groups in the
 *                              descending-width order; unused groups unwritten).
 */
GTQ_API size_t gtq_layout_tile_bytes(int32_t k_bits, int32_t v_bits);

#ifdef __cplusplus
}
#endif
#endif /* GTQ_H */
