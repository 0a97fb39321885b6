// Host-side constant tables of libgtq: Lloyd-Max quantizers of N(0,1) and the
// seeded TurboQuant-MSE rotations, uploaded once per (device, seed).
//
// Lloyd-Max: the b-bit MSE-optimal quantizer of N(0,1) is the fixed point of
// "thresholds are midpoints of adjacent levels" and "each level is the
// conditional mean of its cell".  This file solves that fixed point with
// Newton's method on F(c) = c - centroid(midpoints(c)), whose Jacobian is
// tridiagonal, started from the companding placement sqrt(3) Phi^-1((k+1/2)/N)
// refined by Lloyd alternations.
//
// Rotations: R_m = Q of the Householder QR of an m x m Gaussian matrix, with
// diag(R) > 0.  The Gaussian entry (i, j) takes words 2n, 2n+1 (n = i m + j) of
// the counter-based SplitMix64 stream key = seed ^ (tag << 48) ^ (m << 32)
// (word n = mix(key + (n+1) * 0x9E3779B97F4A7C15), SplitMix64 of Steele, Lea &
// Flood, OOPSLA 2014), and is the Box-Muller cosine variate of
// u1 = ((w >> 11) + 1/2) 2^-53 and u2 = (w' >> 11) 2^-53.
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "gtq_internal.h"

namespace gtq {
namespace {

const double kInvSqrt2 = 0.70710678118654752440;
const double kInvSqrt2Pi = 0.39894228040143267794;

double pdf(double x) { return std::isinf(x) ? 0.0 : kInvSqrt2Pi * std::exp(-0.5 * x * x); }

// P(a < X < b), on the side of zero without cancellation.
double cell_prob(double a, double b) {
  if (a >= 0) return 0.5 * (std::erfc(a * kInvSqrt2) - std::erfc(b * kInvSqrt2));
  return 0.5 * (std::erfc(-b * kInvSqrt2) - std::erfc(-a * kInvSqrt2));
}

double normal_cdf(double x) { return 0.5 * std::erfc(-x * kInvSqrt2); }

double normal_quantile(double p) {  // bisection: plenty for a starting point
  double lo = -40, hi = 40;
  for (int i = 0; i < 200; ++i) {
    double mid = 0.5 * (lo + hi);
    if (normal_cdf(mid) < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

struct LM {
  std::vector<double> c, t;
  double d;
};

void centroid_step(const std::vector<double>& c, std::vector<double>& out) {
  const int n = (int)c.size();
  out.resize(n);
  for (int k = 0; k < n; ++k) {
    double a = k == 0 ? -INFINITY : 0.5 * (c[k - 1] + c[k]);
    double b = k == n - 1 ? INFINITY : 0.5 * (c[k] + c[k + 1]);
    out[k] = (pdf(a) - pdf(b)) / cell_prob(a, b);
  }
}

LM solve_lloyd_max(int bits) {
  LM r;
  if (bits == 0) {
    r.c = {0.0};
    r.d = 1.0;
    return r;
  }
  const int n = 1 << bits;
  std::vector<double> c(n), tmp;
  for (int k = 0; k < n; ++k) c[k] = std::sqrt(3.0) * normal_quantile((k + 0.5) / n);
  for (int it = 0; it < 100; ++it) {
    centroid_step(c, tmp);
    c.swap(tmp);
  }
  // Newton on F_k = c_k - g_k(t_k, t_{k+1}), t_k = (c_{k-1} + c_k) / 2
  std::vector<double> lo(n), di(n), up(n), rhs(n);
  for (int it = 0; it < 60; ++it) {
    double maxstep = 0;
    for (int k = 0; k < n; ++k) {
      double a = k == 0 ? -INFINITY : 0.5 * (c[k - 1] + c[k]);
      double b = k == n - 1 ? INFINITY : 0.5 * (c[k] + c[k + 1]);
      double p = cell_prob(a, b);
      double g = (pdf(a) - pdf(b)) / p;
      double dga = std::isinf(a) ? 0.0 : pdf(a) * (g - a) / p;  // dg/da
      double dgb = std::isinf(b) ? 0.0 : pdf(b) * (b - g) / p;  // dg/db
      lo[k] = -0.5 * dga;
      up[k] = -0.5 * dgb;
      di[k] = 1.0 - 0.5 * dga - 0.5 * dgb;
      rhs[k] = -(c[k] - g);
    }
    // Thomas algorithm
    for (int k = 1; k < n; ++k) {
      double w = lo[k] / di[k - 1];
      di[k] -= w * up[k - 1];
      rhs[k] -= w * rhs[k - 1];
    }
    std::vector<double> x(n);
    x[n - 1] = rhs[n - 1] / di[n - 1];
    for (int k = n - 2; k >= 0; --k) x[k] = (rhs[k] - up[k] * x[k + 1]) / di[k];
    for (int k = 0; k < n; ++k) {
      c[k] += x[k];
      maxstep = std::fmax(maxstep, std::fabs(x[k]));
    }
    if (maxstep < 1e-16) break;
  }
  // the density is symmetric, so is the optimum: c_k = -c_{n-1-k} exactly
  std::vector<double> sym(n);
  for (int k = 0; k < n; ++k) sym[k] = 0.5 * (c[k] - c[n - 1 - k]);
  c = sym;
  r.c = c;
  r.t.resize(n - 1);
  for (int k = 0; k + 1 < n; ++k) r.t[k] = 0.5 * (c[k] + c[k + 1]);
  double s = 0;
  for (int k = 0; k < n; ++k) {
    double a = k == 0 ? -INFINITY : r.t[k - 1];
    double b = k == n - 1 ? INFINITY : r.t[k];
    s += cell_prob(a, b) * c[k] * c[k];
  }
  r.d = 1.0 - s;
  return r;
}

const LM& lloyd_max_cached(int bits) {
  static std::mutex mu;
  static std::map<int, LM> cache;
  std::lock_guard<std::mutex> g(mu);
  auto it = cache.find(bits);
  if (it == cache.end()) it = cache.emplace(bits, solve_lloyd_max(bits)).first;
  return it->second;
}

uint64_t splitmix_word(uint64_t key, uint64_t n) {
  uint64_t z = key + (n + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// R_m into out (row-major m x m)
void make_rotation(uint64_t seed, int tag, int m, double* out) {
  const uint64_t key = seed ^ ((uint64_t)tag << 48) ^ ((uint64_t)m << 32);
  std::vector<double> a((size_t)m * m);  // column-major working copy: a[j*m + i] = G[i][j]
  const double two_pi = 2.0 * M_PI;
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < m; ++j) {
      uint64_t n = (uint64_t)i * m + j;
      double u1 = ((double)(splitmix_word(key, 2 * n) >> 11) + 0.5) * 0x1p-53;
      double u2 = (double)(splitmix_word(key, 2 * n + 1) >> 11) * 0x1p-53;
      a[(size_t)j * m + i] = std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
    }
  // Householder QR: reflectors v_j stored separately, R diagonal in rdiag
  std::vector<std::vector<double>> vs(m);
  std::vector<double> rdiag(m);
  for (int j = 0; j < m; ++j) {
    double* col = &a[(size_t)j * m];
    double norm = 0;
    for (int i = j; i < m; ++i) norm += col[i] * col[i];
    norm = std::sqrt(norm);
    double alpha = col[j] > 0 ? -norm : norm;
    std::vector<double> v(m - j);
    for (int i = j; i < m; ++i) v[i - j] = col[i];
    v[0] -= alpha;
    double vn = 0;
    for (double x : v) vn += x * x;
    if (vn > 0) {
      for (int k = j; k < m; ++k) {  // apply H = I - 2 v v^T / (v^T v) to columns k >= j
        double* ck = &a[(size_t)k * m];
        double dot = 0;
        for (int i = j; i < m; ++i) dot += v[i - j] * ck[i];
        double f = 2.0 * dot / vn;
        for (int i = j; i < m; ++i) ck[i] -= f * v[i - j];
      }
    }
    rdiag[j] = a[(size_t)j * m + j];
    vs[j] = v;
    (void)vn;
  }
  // Q = H_0 H_1 ... H_{m-1}: apply to the identity from the last reflector
  std::vector<double> q((size_t)m * m, 0.0);  // column-major
  for (int i = 0; i < m; ++i) q[(size_t)i * m + i] = 1.0;
  for (int j = m - 1; j >= 0; --j) {
    const std::vector<double>& v = vs[j];
    double vn = 0;
    for (double x : v) vn += x * x;
    if (vn == 0) continue;
    for (int k = 0; k < m; ++k) {
      double* ck = &q[(size_t)k * m];
      double dot = 0;
      for (int i = j; i < m; ++i) dot += v[i - j] * ck[i];
      double f = 2.0 * dot / vn;
      for (int i = j; i < m; ++i) ck[i] -= f * v[i - j];
    }
  }
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < m; ++j) {
      double s = rdiag[j] < 0 ? -1.0 : 1.0;  // make diag(R) > 0
      out[(size_t)i * m + j] = q[(size_t)j * m + i] * s;
    }
}

}  // namespace

int lloyd_max_host(int bits, double* c, double* t, double* d) {
  if (bits < 0 || bits > GTQ_MAX_BITS) return GTQ_ERR_INVALID;
  const LM& r = lloyd_max_cached(bits);
  if (c) std::memcpy(c, r.c.data(), r.c.size() * sizeof(double));
  if (t && !r.t.empty()) std::memcpy(t, r.t.data(), r.t.size() * sizeof(double));
  if (d) *d = r.d;
  return GTQ_OK;
}

int rotation_host(uint64_t seed, int tag, int m, double* out) {
  if (!out || m < 1 || m > 4096) return GTQ_ERR_INVALID;
  make_rotation(seed, tag, m, out);
  return GTQ_OK;
}

int tables_for(int device, uint64_t seed, Tables* out) {
  static std::mutex mu;
  static std::map<std::pair<int, uint64_t>, Tables> cache;
  std::lock_guard<std::mutex> g(mu);
  auto key = std::make_pair(device, seed);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *out = it->second;
    return GTQ_OK;
  }
  // host copies
  std::vector<double> rk(rot_k_total());
  for (int m = 2; m <= kD; m += 2) make_rotation(seed, 0x4B, m, rk.data() + rot_k_offset(m));
  std::vector<double> rv64((size_t)kD * kD);
  make_rotation(seed, 0x56, kD, rv64.data());
  std::vector<float> rv(rv64.begin(), rv64.end());
  std::vector<float> rvt((size_t)kD * kD);
  for (int r = 0; r < kD; ++r)
    for (int d = 0; d < kD; ++d) rvt[(size_t)d * kD + r] = rv[(size_t)r * kD + d];
  std::vector<double> dist(GTQ_MAX_BITS + 1);
  std::vector<float> thr(kThrEntries);
  std::vector<__half> lhi(kLutEntries), llo(kLutEntries);
  for (int w = 0; w <= GTQ_MAX_BITS; ++w) {
    const LM& r = lloyd_max_cached(w);
    dist[w] = r.d;
    if (w == 0) continue;
    for (int k = 0; k < (1 << w) - 1; ++k) thr[thr_base(w) + k] = (float)r.t[k];
    for (int k = 0; k < (1 << w); ++k) {
      __half h = __double2half(r.c[k]);
      lhi[lut_base(w) + k] = h;
      llo[lut_base(w) + k] = __double2half(r.c[k] - (double)__half2float(h));
    }
  }
  // R_V^T as the decode's A fragments: A[dd][r] = R_V[r][dd] for output dims dd
  // (m-tile m: dd = 16 m + ...) and rotated coordinates r (k-tile k); register
  // j of lane (g, t) holds row g + 8 (j & 1), columns 2t + 8 (j >> 1) and the
  // next one (low half first), as fp16 hi and the fp16 remainder lo
  std::vector<uint32_t> rvf((size_t)8 * 8 * 32 * 8);
  for (int mt = 0; mt < 8; ++mt)
    for (int kt = 0; kt < 8; ++kt)
      for (int lane = 0; lane < 32; ++lane)
        for (int j = 0; j < 4; ++j) {
          const int dd = 16 * mt + (lane >> 2) + 8 * (j & 1);
          const int r = 16 * kt + 2 * (lane & 3) + 8 * (j >> 1);
          uint32_t wh = 0, wl = 0;
          for (int e = 0; e < 2; ++e) {
            const float v = rv[(size_t)(r + e) * kD + dd];
            const __half hv = __float2half_rn(v);
            const __half lv = __float2half_rn(v - __half2float(hv));
            uint16_t uh, ul;
            std::memcpy(&uh, &hv, 2);
            std::memcpy(&ul, &lv, 2);
            wh |= (uint32_t)uh << (16 * e);
            wl |= (uint32_t)ul << (16 * e);
          }
          const size_t base = (((size_t)mt * 8 + kt) * 32 + lane) * 8;
          rvf[base + j] = wh;
          rvf[base + 4 + j] = wl;
        }
  // decode lookup-table image (layout: gtq_internal.h, kTab*)
  std::vector<uint32_t> img(kDecodeImageBytes / 4, 0u);
  auto bits16 = [](__half h) { uint16_t u; std::memcpy(&u, &h, 2); return (uint32_t)u; };
  auto hi = [&](int w, int c) { return bits16(lhi[lut_base(w) + c]); };
  auto lo = [&](int w, int c) { return bits16(llo[lut_base(w) + c]); };
  for (int w = 1; w <= 4; ++w)
    for (int idx = 0; idx < (1 << (2 * w)); ++idx) {
      const int c0 = idx & ((1 << w) - 1), c1 = idx >> w;
      const uint32_t vh = hi(w, c0) | (hi(w, c1) << 16), vl = lo(w, c0) | (lo(w, c1) << 16);
      for (int cp = 0; cp < 16; ++cp) {  // P16: {hi half2, lo half2} per lane pair
        img[(kTabP16(w) + idx * 128 + cp * 8) / 4] = vh;
        img[(kTabP16(w) + idx * 128 + cp * 8) / 4 + 1] = vl;
      }
      if (w <= 3)
        for (int lane = 0; lane < 32; ++lane) img[(kTabP32(w) + idx * 128 + lane * 4) / 4] = vh;
    }
  for (int w = 5; w <= 6; ++w)
    for (int c = 0; c < (1 << w); ++c)
      for (int lane = 0; lane < 32; ++lane)
        img[(kTabS32(w) + c * 128 + lane * 4) / 4] = hi(w, c) | (lo(w, c) << 16);
  for (int w = 1; w <= GTQ_MAX_BITS; ++w)
    for (int c = 0; c < (1 << w); ++c)
      img[(kTabSS + kSingleOff(w)) / 4 + c] = hi(w, c) | (lo(w, c) << 16);
  Tables t{};
  auto up = [](void** dst, const void* src, size_t bytes) -> cudaError_t {
    cudaError_t e = cudaMalloc(dst, bytes);
    if (e != cudaSuccess) return e;
    return cudaMemcpy(*dst, src, bytes, cudaMemcpyHostToDevice);
  };
  int prev = 0;
  cudaGetDevice(&prev);
  if (cudaSetDevice(device) != cudaSuccess) return GTQ_ERR_CUDA;
  cudaError_t e = up((void**)&t.rot_k, rk.data(), rk.size() * sizeof(double));
  if (e == cudaSuccess) e = up((void**)&t.rot_v, rv.data(), rv.size() * sizeof(float));
  if (e == cudaSuccess) e = up((void**)&t.rot_vt, rvt.data(), rvt.size() * sizeof(float));
  if (e == cudaSuccess) e = up((void**)&t.rv_frag, rvf.data(), rvf.size() * sizeof(uint32_t));
  if (e == cudaSuccess) e = up((void**)&t.dist, dist.data(), dist.size() * sizeof(double));
  if (e == cudaSuccess) e = up((void**)&t.thr, thr.data(), thr.size() * sizeof(float));
  if (e == cudaSuccess) e = up((void**)&t.dec_image, img.data(), img.size() * sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMalloc((void**)&t.rv_image, b_image_bytes());
  if (e == cudaSuccess) e = build_b_images(t.rot_v, 1, 0, t.rv_image, 0);
  if (e == cudaSuccess) e = cudaMalloc((void**)&t.code_lut, kCodeLutBytes);
  if (e == cudaSuccess) e = build_code_lut(t.thr, t.code_lut, 0);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) {
    int ok = 0;
    e = cudaMemcpy(&ok, t.code_lut + kCodeLutOkOffset, sizeof(ok), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && ok != 1) {
      cudaSetDevice(prev);
      set_last_error("code lookup table: two thresholds share a cell");
      return GTQ_ERR_CUDA;
    }
  }
  cudaSetDevice(prev);
  if (e != cudaSuccess) return e == cudaErrorMemoryAllocation ? GTQ_ERR_OOM : GTQ_ERR_CUDA;
  cache[key] = t;
  *out = t;
  return GTQ_OK;
}

}  // namespace gtq
