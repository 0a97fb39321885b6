// C ABI of libgtq: argument validation, plan lifetime and kernel launches.
// Every entry point returns a GTQ_* code; nothing throws across the boundary.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "gtq_internal.h"

using namespace gtq;

namespace {

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int check_config(const gtq_config* c, bool need_128) {
  if (!c) return GTQ_ERR_INVALID;
  if (c->batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1) return GTQ_ERR_INVALID;
  if (c->n_q_heads % c->n_kv_heads) return GTQ_ERR_INVALID;
  // heads are the grid's y extent in the energy and quantize launches
  if ((int64_t)c->batch * c->n_kv_heads > 65535) return GTQ_ERR_UNSUPPORTED;
  if (c->n_q_heads / c->n_kv_heads > kMaxGq) return GTQ_ERR_UNSUPPORTED;
  if (c->head_dim < 4 || c->head_dim > kD || (c->head_dim & 1)) return GTQ_ERR_UNSUPPORTED;
  if (need_128 && c->head_dim != kD) return GTQ_ERR_UNSUPPORTED;
  if (c->max_bits < 1 || c->max_bits > GTQ_MAX_BITS) return GTQ_ERR_INVALID;
  if (c->k_bits < 1 || c->k_bits > c->max_bits) return GTQ_ERR_INVALID;
  if (c->v_bits < 0 || c->v_bits > GTQ_MAX_BITS) return GTQ_ERR_INVALID;  // 0: K-only
  if (c->rope_pairing != GTQ_PAIRING_HALF && c->rope_pairing != GTQ_PAIRING_INTERLEAVED)
    return GTQ_ERR_INVALID;
  if (c->in_dtype != GTQ_DTYPE_FP16 && c->in_dtype != GTQ_DTYPE_FP32) return GTQ_ERR_INVALID;
  if (c->reserved != 0) return GTQ_ERR_INVALID;
  if (c->t_capacity < 1 || c->t_capacity > (int64_t(1) << 40)) return GTQ_ERR_INVALID;
  return GTQ_OK;
}

thread_local char g_last_error[256] = "";

int cuda_code(cudaError_t e) {
  if (e == cudaSuccess) return GTQ_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e),
           cudaGetErrorString(e));
  return e == cudaErrorMemoryAllocation ? GTQ_ERR_OOM : GTQ_ERR_CUDA;
}

void release(gtq_plan* p) {
  if (!p) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(p->device);
  cudaFree(p->d_energy);
  cudaFree(p->d_bits);
  cudaFree(p->d_meta);
  cudaFree(p->d_mrow);
  cudaFree(p->d_rotpack);
  cudaFree(p->d_bimg);
  cudaFree(p->d_partials);
  cudaFree(p->d_tickets);
  cudaFree(p->d_status);
  cudaSetDevice(prev);
  delete p;
}

// common plan construction: validation done by the caller
int make_plan(const gtq_config* cfg, gtq_plan** out) {
  gtq_plan* p = new (std::nothrow) gtq_plan();
  if (!p) return GTQ_ERR_OOM;
  p->cfg = *cfg;
  if (cudaGetDevice(&p->device) != cudaSuccess) {
    delete p;
    return GTQ_ERR_CUDA;
  }
  cudaDeviceGetAttribute(&p->n_sms, cudaDevAttrMultiProcessorCount, p->device);
  p->n_heads = cfg->batch * cfg->n_kv_heads;
  p->n_blocks = cfg->head_dim / 2;
  p->g_q = cfg->n_q_heads / cfg->n_kv_heads;
  p->n_qs = (p->g_q + kQSlice - 1) / kQSlice;
  p->n_units = p->n_heads * p->n_qs;
  p->n_tiles = (cfg->t_capacity + kTile - 1) / kTile;
  p->tile_bytes = gtq_layout_tile_bytes(cfg->k_bits, cfg->v_bits);
  p->packed_bytes = (size_t)p->n_heads * p->n_tiles * p->tile_bytes;
  int rc = tables_for(p->device, cfg->seed, &p->tab);
  if (rc != GTQ_OK) {
    delete p;
    return rc;
  }
  const size_t H = p->n_heads;
  cudaError_t e = cudaSuccess;
  auto alloc = [&](void** ptr, size_t bytes) {
    if (e == cudaSuccess) e = cudaMalloc(ptr, bytes);
  };
  alloc((void**)&p->d_energy, H * p->n_blocks * sizeof(double));
  alloc((void**)&p->d_bits, H * p->n_blocks);
  alloc((void**)&p->d_meta, H * sizeof(HeadMeta));
  alloc((void**)&p->d_mrow, H * kD * kD * sizeof(float));
  alloc((void**)&p->d_rotpack, H * kRotPackBytes);
  if (cfg->head_dim == kD) alloc((void**)&p->d_bimg, H * b_image_bytes());
  const size_t U = p->n_units;
  alloc((void**)&p->d_partials, U * (size_t)PartialSlots(decode_split_cap(p->n_sms, p->n_units)).total *
                                    8 * kPartialStride * sizeof(float));
  alloc((void**)&p->d_tickets, U * kTicketStride * sizeof(unsigned));
  alloc((void**)&p->d_status, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(p->d_tickets, 0, U * kTicketStride * sizeof(unsigned));
  if (e == cudaSuccess) e = cudaMemset(p->d_status, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(p->d_meta, 0, H * sizeof(HeadMeta));
  if (e != cudaSuccess) {
    release(p);
    return cuda_code(e);
  }
  *out = p;
  return GTQ_OK;
}

// a layout's pointers and sizes (its contents live on the device)
int check_layout(const gtq_seq_layout* lay, int64_t T) {
  if (!lay) return GTQ_OK;
  if (lay->seq_lens_dev && !aligned(lay->seq_lens_dev, 4)) return GTQ_ERR_INVALID;
  if (lay->block_table_dev) {
    if (!aligned(lay->block_table_dev, 4) || lay->max_blocks < 1) return GTQ_ERR_INVALID;
    if ((T + kTile - 1) / kTile > lay->max_blocks) return GTQ_ERR_INVALID;
  }
  return GTQ_OK;
}

}  // namespace

namespace gtq {
SeqMap seq_map(const gtq_plan* p, const gtq_seq_layout* lay) {
  SeqMap m;
  m.hkv = p->cfg.n_kv_heads;
  m.n_tiles = p->n_tiles;
  m.tile_bytes = (int64_t)p->tile_bytes;
  if (lay) {
    m.seq_lens = lay->seq_lens_dev;
    m.table = lay->block_table_dev;
    m.max_blocks = lay->block_table_dev ? lay->max_blocks : 0;
  }
  return m;
}
void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }
int record_cuda_error(cudaError_t e) { return cuda_code(e); }
}  // namespace gtq

extern "C" {

size_t gtq_layout_tile_bytes(int32_t k_bits, int32_t v_bits) {
  if (k_bits < 1 || k_bits > GTQ_MAX_BITS || v_bits < 0 || v_bits > GTQ_MAX_BITS) return 0;
  return (size_t)key_norm_offset(k_bits, v_bits) + 128 * kMaxGroups;
}

int gtq_alloc_bits(const gtq_config* cfg, const void* k_dev, int64_t T, const int64_t k_strides[4],
                   void* stream, gtq_plan** out) {
  return gtq_alloc_bits_ex(cfg, k_dev, T, k_strides, nullptr, stream, out);
}

int gtq_alloc_bits_ex(const gtq_config* cfg, const void* k_dev, int64_t T,
                      const int64_t k_strides[4], const gtq_seq_layout* lay, void* stream,
                      gtq_plan** out) {
  if (!out || !k_dev || !k_strides) return GTQ_ERR_INVALID;
  if (lay && lay->seq_lens_dev && !aligned(lay->seq_lens_dev, 4)) return GTQ_ERR_INVALID;
  int rc = check_config(cfg, false);
  if (rc != GTQ_OK) return rc;
  if (cfg->head_dim % 8) return GTQ_ERR_UNSUPPORTED;  // energy pass reads 8-dim vectors
  if (T < 1 || T > cfg->t_capacity) return GTQ_ERR_INVALID;
  const int esz = cfg->in_dtype == GTQ_DTYPE_FP16 ? 2 : 4;
  if (k_strides[3] != 1 || !aligned(k_dev, 16)) return GTQ_ERR_INVALID;
  for (int i = 0; i < 3; ++i)
    if (k_strides[i] < 0 || (k_strides[i] * esz) % 16) return GTQ_ERR_INVALID;
  gtq_plan* p = nullptr;
  rc = make_plan(cfg, &p);
  if (rc != GTQ_OK) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_energy(p, k_dev, T, k_strides, lay ? lay->seq_lens_dev : nullptr, s);
  if (e == cudaSuccess) e = launch_greedy_and_meta(p, s);
  if (e != cudaSuccess) {
    cudaStreamSynchronize(s);
    release(p);
    return cuda_code(e);
  }
  *out = p;
  return GTQ_OK;
}

int gtq_alloc_bits_from_energy(const gtq_config* cfg, const double* host_energy, gtq_plan** out) {
  if (!out || !host_energy) return GTQ_ERR_INVALID;
  int rc = check_config(cfg, false);
  if (rc != GTQ_OK) return rc;
  gtq_plan* p = nullptr;
  rc = make_plan(cfg, &p);
  if (rc != GTQ_OK) return rc;
  cudaError_t e = cudaMemcpy(p->d_energy, host_energy,
                             (size_t)p->n_heads * p->n_blocks * sizeof(double),
                             cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = launch_greedy_and_meta(p, 0);
  if (e == cudaSuccess) e = cudaStreamSynchronize(0);
  if (e != cudaSuccess) {
    release(p);
    return cuda_code(e);
  }
  *out = p;
  return GTQ_OK;
}

int gtq_quantize_pack(gtq_plan* plan, const void* k_dev, const void* v_dev,
                      const int64_t strides[4], int64_t t0, int64_t n_tokens, void* packed_dev,
                      size_t packed_bytes, void* stream) {
  return gtq_quantize_pack_ex(plan, k_dev, v_dev, strides, t0, n_tokens, packed_dev, packed_bytes,
                              nullptr, stream);
}

int gtq_quantize_pack_ex(gtq_plan* plan, const void* k_dev, const void* v_dev,
                         const int64_t strides[4], int64_t t0, int64_t n_tokens, void* packed_dev,
                         size_t packed_bytes, const gtq_seq_layout* lay, void* stream) {
  if (!plan || !k_dev || !strides || !packed_dev) return GTQ_ERR_INVALID;
  // values: coded plans need them, K-only plans (v_bits 0) take none
  if ((v_dev != nullptr) != (plan->cfg.v_bits > 0)) return GTQ_ERR_INVALID;
  if (!v_dev) v_dev = k_dev;  // (never read)
  if (plan->cfg.head_dim != kD) return GTQ_ERR_UNSUPPORTED;
  const bool tail = t0 == GTQ_T0_TAIL;
  if (tail && !(lay && lay->seq_lens_dev)) return GTQ_ERR_INVALID;
  if (tail) t0 = 0;  // the range checks below then bound n_tokens by the capacity
  if (t0 < 0 || n_tokens < 1 || t0 + n_tokens > plan->cfg.t_capacity) return GTQ_ERR_INVALID;
  const bool paged = lay && lay->block_table_dev;
  const size_t need = paged ? (size_t)plan->cfg.n_kv_heads * plan->tile_bytes : plan->packed_bytes;
  if (packed_bytes < need || !aligned(packed_dev, 16)) return GTQ_ERR_INVALID;
  if (check_layout(lay, tail ? plan->cfg.t_capacity : t0 + n_tokens) != GTQ_OK)
    return GTQ_ERR_INVALID;
  const int esz = plan->cfg.in_dtype == GTQ_DTYPE_FP16 ? 2 : 4;
  if (strides[3] != 1 || !aligned(k_dev, esz) || !aligned(v_dev, esz)) return GTQ_ERR_INVALID;
  for (int i = 0; i < 3; ++i)
    if (strides[i] < 0) return GTQ_ERR_INVALID;
  SeqMap sm = seq_map(plan, lay);
  sm.tail = tail ? 1 : 0;
  return cuda_code(launch_quantize(plan, k_dev, v_dev, strides, t0, n_tokens,
                                   (uint8_t*)packed_dev, sm, (cudaStream_t)stream));
}

int gtq_decode_attn(gtq_plan* plan, const void* packed_dev, int64_t T, const void* q_dev,
                    int32_t q_dtype, float* out_dev, void* stream) {
  return gtq_decode_attn_ex(plan, packed_dev, T, nullptr, q_dev, q_dtype, out_dev, stream);
}

int gtq_decode_attn_ex(gtq_plan* plan, const void* packed_dev, int64_t T,
                       const gtq_seq_layout* lay, const void* q_dev, int32_t q_dtype,
                       float* out_dev, void* stream) {
  return gtq_decode_attn_full(plan, packed_dev, T, lay, nullptr, q_dev, q_dtype, out_dev, stream);
}

int gtq_decode_attn_full(gtq_plan* plan, const void* packed_dev, int64_t T,
                         const gtq_seq_layout* lay, const gtq_fp16_kv* kv, const void* q_dev,
                         int32_t q_dtype, float* out_dev, void* stream) {
  if (!plan || !packed_dev || !q_dev || !out_dev) return GTQ_ERR_INVALID;
  Fp16Kv f;
  const bool konly = plan->cfg.v_bits == 0;
  if (konly != (kv && kv->v_dev)) return GTQ_ERR_INVALID;  // values: coded xor fp16
  if (konly) {
    if (!aligned(kv->v_dev, 16) || kv->v_strides[3] != 1) return GTQ_ERR_INVALID;
    for (int i = 0; i < 3; ++i)
      if (kv->v_strides[i] < 0 || kv->v_strides[i] % 8) return GTQ_ERR_INVALID;
    f.v = (const __half*)kv->v_dev;
    for (int i = 0; i < 4; ++i) f.vs[i] = kv->v_strides[i];
  }
  if (kv && kv->recent_len != 0) {
    if (kv->recent_len < 0 || kv->recent_len > kMaxWindow) return GTQ_ERR_INVALID;
    if (!kv->recent_k_dev || !kv->recent_v_dev || !aligned(kv->recent_k_dev, 16) ||
        !aligned(kv->recent_v_dev, 16) || kv->recent_strides[3] != 1 ||
        !aligned(kv->recent_lens_dev, 4))
      return GTQ_ERR_INVALID;
    for (int i = 0; i < 3; ++i)
      if (kv->recent_strides[i] < 0 || kv->recent_strides[i] % 8) return GTQ_ERR_INVALID;
    f.rk = (const __half*)kv->recent_k_dev;
    f.rv = (const __half*)kv->recent_v_dev;
    for (int i = 0; i < 4; ++i) f.rs[i] = kv->recent_strides[i];
    f.rlens = kv->recent_lens_dev;
    f.rlen = kv->recent_len;
  }
  if (plan->cfg.head_dim != kD) return GTQ_ERR_UNSUPPORTED;
  if (T < 1 || T > plan->cfg.t_capacity) return GTQ_ERR_INVALID;
  if (q_dtype != GTQ_DTYPE_FP16 && q_dtype != GTQ_DTYPE_FP32) return GTQ_ERR_INVALID;
  if (!aligned(packed_dev, 16) || !aligned(q_dev, 16) || !aligned(out_dev, 16))
    return GTQ_ERR_INVALID;
  if (check_layout(lay, T) != GTQ_OK) return GTQ_ERR_INVALID;
  return cuda_code(launch_decode(plan, (const uint8_t*)packed_dev, T, q_dev, q_dtype, out_dev,
                                 seq_map(plan, lay), f, (cudaStream_t)stream));
}

int gtq_free(gtq_plan* plan) {
  if (!plan) return GTQ_OK;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(plan->device);
  cudaError_t e = cudaDeviceSynchronize();
  cudaSetDevice(prev);
  release(plan);
  return cuda_code(e);
}

size_t gtq_packed_bytes(const gtq_plan* plan) { return plan ? plan->packed_bytes : 0; }

int gtq_get_bits(gtq_plan* plan, uint8_t* host_bits, void* stream) {
  if (!plan || !host_bits) return GTQ_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(host_bits, plan->d_bits, (size_t)plan->n_heads * plan->n_blocks,
                                  cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_code(e);
}

int gtq_get_energy(gtq_plan* plan, double* host_energy, void* stream) {
  if (!plan || !host_energy) return GTQ_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(host_energy, plan->d_energy,
                                  (size_t)plan->n_heads * plan->n_blocks * sizeof(double),
                                  cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_code(e);
}

size_t gtq_plan_device_bytes(const gtq_plan* plan) {
  if (!plan) return 0;
  const size_t H = plan->n_heads, U = plan->n_units;
  size_t b = H * plan->n_blocks * sizeof(double) + H * plan->n_blocks + H * sizeof(HeadMeta) +
             H * kD * kD * sizeof(float) + H * kRotPackBytes +
             U * (size_t)PartialSlots(decode_split_cap(plan->n_sms, plan->n_units)).total * 8 *
                 kPartialStride * sizeof(float) +
             U * kTicketStride * sizeof(unsigned) + sizeof(int);
  if (plan->cfg.head_dim == kD) b += H * b_image_bytes();
  return b;
}

int gtq_raise_status(gtq_plan* plan, int32_t code) {
  if (!plan) return GTQ_ERR_INVALID;
  int bit = 0;
  if (code == GTQ_ERR_TIMEOUT) bit = kStatusTimeout;
  else if (code == GTQ_ERR_OVERFLOW) bit = kStatusOverflow;
  else return GTQ_ERR_INVALID;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaError_t e = cudaSetDevice(plan->device);
  int v = 0;
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&v, plan->d_status, sizeof(int), cudaMemcpyDeviceToHost);
  v |= bit;
  if (e == cudaSuccess) e = cudaMemcpy(plan->d_status, &v, sizeof(int), cudaMemcpyHostToDevice);
  cudaSetDevice(prev);
  return cuda_code(e);
}

int gtq_status(gtq_plan* plan) {
  if (!plan) return GTQ_ERR_INVALID;
  int v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&v, plan->d_status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(plan->d_status, 0, sizeof(int));
  if (e != cudaSuccess) return GTQ_ERR_CUDA;
  if (v & kStatusLayout) {
    set_last_error("decode kernel: shared-memory window above the planned layout");
    return GTQ_ERR_CUDA;
  }
  if (v & kStatusTimeout) return GTQ_ERR_TIMEOUT;
  if (v & kStatusOverflow) return GTQ_ERR_OVERFLOW;
  return GTQ_OK;
}

const char* gtq_last_error(void) { return g_last_error; }

const char* gtq_strerror(int code) {
  switch (code) {
    case GTQ_OK: return "ok";
    case GTQ_ERR_INVALID: return "invalid argument";
    case GTQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case GTQ_ERR_CUDA: return "CUDA runtime error";
    case GTQ_ERR_OOM: return "device out of memory";
    case GTQ_ERR_TIMEOUT: return "bounded device wait expired";
    case GTQ_ERR_OVERFLOW: return "norm above the fp16 range (clamped)";
    case GTQ_ERR_STATE: return "plan not ready";
    default: return "unknown error";
  }
}

int gtq_lloyd_max(int32_t bits, double* centroids, double* thresholds, double* distortion) {
  return lloyd_max_host(bits, centroids, thresholds, distortion);
}

int gtq_rotation(uint64_t seed, int32_t tag, int32_t m, double* out) {
  if (tag != 0x4B && tag != 0x56) return GTQ_ERR_INVALID;
  if (tag == 0x4B && (m < 2 || m > kD || (m & 1))) return GTQ_ERR_INVALID;
  if (tag == 0x56 && m != kD) return GTQ_ERR_INVALID;
  return rotation_host(seed, tag, m, out);
}

}  // extern "C"
