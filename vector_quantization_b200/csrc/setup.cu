// Host-side construction of a codec handle: Lloyd-Max codebook, rotation,
// QJL matrix and RoPE tables, all in float64, then uploaded to the device.
//
// [TurboQuant] "Principe de fonctionnement", Étape 1: a data-oblivious random
// rotation followed by a standard high-quality scalar quantizer per
// coordinate, whose boundaries and levels come from Lloyd-Max (comments
// section); "QJL": Gaussian Johnson-Lindenstrauss projection reduced to sign
// bits.  [NSNQuant] Méthodologie §2: randomized Hadamard transform.
// [TurboESM] §2.A: RoPE applied before the rotation.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <limits>
#include <new>
#include <vector>

#include "tq_internal.h"

namespace {

// ---------------------------------------------------------------------------
// Regularized incomplete beta function.  Continued-fraction expansion of
// I_x(a, b) evaluated with the modified Lentz method (the classical route,
// e.g. Abramowitz & Stegun 26.5.8; Lentz 1976).  Returns I and its
// complement, each accurate where it is the smaller of the two.
// ---------------------------------------------------------------------------
double beta_continued_fraction(double a, double b, double x) {
  const double tiny = 1e-300;
  const double eps = 1e-17;
  const double ab = a + b, ap = a + 1.0, am = a - 1.0;
  double c = 1.0;
  double dd = 1.0 - ab * x / ap;
  if (std::fabs(dd) < tiny) dd = tiny;
  dd = 1.0 / dd;
  double f = dd;
  for (int k = 1; k <= 200000; ++k) {
    const double k2 = 2.0 * k;
    // even step
    double num = k * (b - k) * x / ((am + k2) * (a + k2));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    f *= dd * c;
    // odd step
    num = -(a + k) * (ab + k) * x / ((a + k2) * (ap + k2));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    const double step = dd * c;
    f *= step;
    if (std::fabs(step - 1.0) < eps) break;
  }
  return f;
}

void incomplete_beta(double a, double b, double x, double* I, double* Ic) {
  if (x <= 0.0) { *I = 0.0; *Ic = 1.0; return; }
  if (x >= 1.0) { *I = 1.0; *Ic = 0.0; return; }
  const double front = std::exp(std::lgamma(a + b) - std::lgamma(a) - std::lgamma(b) +
                                a * std::log(x) + b * std::log1p(-x));
  if (x < (a + 1.0) / (a + b + 2.0)) {
    *I = front * beta_continued_fraction(a, b, x) / a;
    *Ic = 1.0 - *I;
  } else {
    *Ic = front * beta_continued_fraction(b, a, 1.0 - x) / b;
    *I = 1.0 - *Ic;
  }
}

// Density of one coordinate T of a uniform point on S^{d-1}:
// f(t) = C_d (1 - t^2)^((d-3)/2).  T^2 ~ Beta(1/2, (d-1)/2).
double log_cd(int d) {
  return std::lgamma(0.5 * d) - 0.5 * std::log(M_PI) - std::lgamma(0.5 * (d - 1));
}

// P(a <= T < b) for 0 <= a <= b <= 1.
double coord_mass(double a, double b, int d) {
  const double k = 0.5 * (d - 1);
  double Ia, Ica, Ib, Icb;
  incomplete_beta(0.5, k, a * a, &Ia, &Ica);
  incomplete_beta(0.5, k, b * b, &Ib, &Icb);
  if (Ia <= 0.5) return 0.5 * (Ib - Ia);
  return 0.5 * (Ica - Icb);
}

// Integral of t f(t) over [a, b]: C_d [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)] / (d-1).
double coord_first_moment(double a, double b, int d) {
  const double k = 0.5 * (d - 1);
  const double lc = log_cd(d) - std::log(static_cast<double>(d - 1));
  const double pa = a < 1.0 ? std::exp(lc + k * std::log1p(-a * a)) : 0.0;
  const double pb = b < 1.0 ? std::exp(lc + k * std::log1p(-b * b)) : 0.0;
  return pa - pb;
}

// Lloyd-Max iteration on the positive half (the law is symmetric, the middle
// threshold is 0).  Stops when no level moves by 1e-14 of the largest level,
// or when the iteration has settled on the evaluation noise floor.
bool lloyd_max_levels(int d, int bits, std::vector<double>* levels,
                      std::vector<double>* thresholds) {
  const int L = 1 << (bits - 1);
  const double spread = std::fmin(1.0, 3.0 / std::sqrt(static_cast<double>(d)));
  std::vector<double> c(L), t(L + 1), cn(L);
  for (int j = 0; j < L; ++j) c[j] = (j + 0.5) / L * spread;
  double best = std::numeric_limits<double>::infinity();
  int stalled = 0;
  bool done = false;
  for (int it = 0; it < 200000 && !done; ++it) {
    t[0] = 0.0;
    t[L] = 1.0;
    for (int j = 1; j < L; ++j) t[j] = 0.5 * (c[j - 1] + c[j]);
    double moved = 0.0, top = 0.0;
    for (int j = 0; j < L; ++j) {
      cn[j] = coord_first_moment(t[j], t[j + 1], d) / coord_mass(t[j], t[j + 1], d);
      moved = std::fmax(moved, std::fabs(cn[j] - c[j]));
      top = std::fmax(top, std::fabs(cn[j]));
    }
    c = cn;
    moved /= top;
    if (moved <= 1e-14) done = true;
    stalled = moved >= best ? stalled + 1 : 0;
    best = std::fmin(best, moved);
    if (best < 1e-10 && stalled > 200) done = true;
  }
  if (!done) return false;
  levels->assign(2 * L, 0.0);
  for (int j = 0; j < L; ++j) {
    (*levels)[L + j] = c[j];
    (*levels)[L - 1 - j] = -c[j];
  }
  thresholds->assign(2 * L - 1, 0.0);
  for (int j = 0; j + 1 < 2 * L; ++j) (*thresholds)[j] = 0.5 * ((*levels)[j] + (*levels)[j + 1]);
  return true;
}

// Subsets of code bits whose +-1 products span an odd-symmetric codebook:
// bits 1 -> {0}; bits 2 -> {1}, {0}; bits 3 -> {2}, {1}, {0}, {0,1,2}.
int plane_subsets(int bits, unsigned* subsets) {
  if (bits == 1) { subsets[0] = 1u; return 1; }
  if (bits == 2) { subsets[0] = 2u; subsets[1] = 1u; return 2; }
  subsets[0] = 4u; subsets[1] = 2u; subsets[2] = 1u; subsets[3] = 7u;
  return 4;
}

float round_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return f;  // NaN stays NaN
  const uint32_t lsb = (u >> 16) & 1u;
  u = (u + 0x7fffu + lsb) & 0xffff0000u;
  std::memcpy(&f, &u, 4);
  return f;
}

// Householder QR of an n x n matrix G (row-major), returning Pi = Q diag(sign(diag R))
// (row-major): the Haar-distributed orthogonal factor with positive R diagonal.
void haar_from_gaussian(const double* G, int n, std::vector<double>* pi) {
  std::vector<double> A(static_cast<size_t>(n) * n);  // column-major working copy
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) A[i + static_cast<size_t>(j) * n] = G[static_cast<size_t>(i) * n + j];
  std::vector<double> beta(n, 0.0), rdiag(n, 0.0);
  for (int k = 0; k < n; ++k) {
    double* x = &A[k + static_cast<size_t>(k) * n];
    const int len = n - k;
    double nrm2 = 0.0;
    for (int i = 0; i < len; ++i) nrm2 += x[i] * x[i];
    const double nrm = std::sqrt(nrm2);
    const double alpha = x[0] >= 0.0 ? -nrm : nrm;  // x -> alpha e_1
    rdiag[k] = alpha;
    x[0] -= alpha;                                    // x now holds v
    double vv = 0.0;
    for (int i = 0; i < len; ++i) vv += x[i] * x[i];
    beta[k] = vv > 0.0 ? 2.0 / vv : 0.0;
    const double bk = beta[k];
#pragma omp parallel for schedule(static)
    for (int j = k + 1; j < n; ++j) {
      double* col = &A[k + static_cast<size_t>(j) * n];
      double w = 0.0;
      for (int i = 0; i < len; ++i) w += x[i] * col[i];
      w *= bk;
      for (int i = 0; i < len; ++i) col[i] -= w * x[i];
    }
  }
  // Q = H_0 H_1 ... H_{n-1} applied to the identity, accumulated backwards.
  std::vector<double> Q(static_cast<size_t>(n) * n, 0.0);  // column-major
  for (int i = 0; i < n; ++i) Q[i + static_cast<size_t>(i) * n] = 1.0;
  for (int k = n - 1; k >= 0; --k) {
    const double* v = &A[k + static_cast<size_t>(k) * n];
    const int len = n - k;
    const double bk = beta[k];
#pragma omp parallel for schedule(static)
    for (int j = 0; j < n; ++j) {
      double* col = &Q[k + static_cast<size_t>(j) * n];
      double w = 0.0;
      for (int i = 0; i < len; ++i) w += v[i] * col[i];
      w *= bk;
      for (int i = 0; i < len; ++i) col[i] -= w * v[i];
    }
  }
  pi->assign(static_cast<size_t>(n) * n, 0.0);
  for (int j = 0; j < n; ++j) {
    const double s = rdiag[j] < 0.0 ? -1.0 : 1.0;
    for (int i = 0; i < n; ++i)
      (*pi)[static_cast<size_t>(i) * n + j] = s * Q[i + static_cast<size_t>(j) * n];
  }
}

template <typename T>
int upload(T** dst, const T* src, size_t count) {
  if (count == 0) return TQ_OK;
  if (cudaMalloc(reinterpret_cast<void**>(dst), count * sizeof(T)) != cudaSuccess) {
    cudaGetLastError();
    return TQ_ENOMEM;
  }
  if (cudaMemcpy(*dst, src, count * sizeof(T), cudaMemcpyHostToDevice) != cudaSuccess) return TQ_ECUDA;
  return TQ_OK;
}

void release(tq_rotation* h) {
  if (!h) return;
  cudaFree(h->d_levels);
  cudaFree(h->d_thresholds);
  cudaFree(h->d_signs);
  cudaFree(h->d_pi);
  cudaFree(h->d_s);
  cudaFree(h->d_st);
  cudaFree(h->d_s_op);
  cudaFree(h->d_hd_f16);
  cudaFree(h->d_hd_bf16);
  cudaFree(h->d_enc_epi);
  cudaFree(h->d_pi_hi);
  cudaFree(h->d_pi_lo);
  cudaFree(h->d_s_bf16);
  cudaFree(h->d_rope_hi);
  cudaFree(h->d_rope_lo);
  delete h;
}

// ---------------------------------------------------------------------------
// Seeded draws of a handle: the counter-based generator Philox4x32-10
// (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
// SC 2011).  Ten rounds; a round multiplies counter words 0 and 2 by two
// fixed 32-bit constants, keeps the low halves as the new words 3 and 1, and
// XORs the high halves with the other two words and the key; the key steps
// by two Weyl constants between rounds.  How a handle uses it:
//   key = (seed mod 2^32, seed >> 32); counter = (i mod 2^32, i >> 32,
//   stream, 0), stream 0 for the sign diagonal D, 1 for the QJL matrix S,
//   2 for the Gaussian matrix behind a dense rotation.
//   D_i = -1 when the top bit of word 0 of block i is set, else +1.
//   Gaussians in pairs: block p gives two uniforms
//   u = ((w0 >> 6) 2^26 + (w1 >> 6) + 1/2) / 2^52 (words 0-1, then 2-3),
//   exact in double and strictly inside (0, 1); then Box-Muller,
//   r = sqrt(-2 ln u1), z_2p = r cos(2 pi u2), z_2p+1 = r sin(2 pi u2).
// ---------------------------------------------------------------------------
struct Philox4 {
  uint32_t w[4];
};

Philox4 philox4x32_10(uint64_t index, uint32_t stream, uint64_t seed) {
  uint32_t c0 = static_cast<uint32_t>(index), c1 = static_cast<uint32_t>(index >> 32), c2 = stream, c3 = 0;
  uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t prod_a = static_cast<uint64_t>(0xD2511F53u) * c0;
    const uint64_t prod_b = static_cast<uint64_t>(0xCD9E8D57u) * c2;
    const uint32_t n0 = static_cast<uint32_t>(prod_b >> 32) ^ c1 ^ k0;
    const uint32_t n1 = static_cast<uint32_t>(prod_b);
    const uint32_t n2 = static_cast<uint32_t>(prod_a >> 32) ^ c3 ^ k1;
    const uint32_t n3 = static_cast<uint32_t>(prod_a);
    c0 = n0;
    c1 = n1;
    c2 = n2;
    c3 = n3;
  }
  return Philox4{{c0, c1, c2, c3}};
}

constexpr uint32_t kStreamSigns = 0, kStreamQjl = 1, kStreamDense = 2;

double uniform_from_words(uint32_t hi, uint32_t lo) {
  const double a = static_cast<double>(hi >> 6), b = static_cast<double>(lo >> 6);
  return (a * 67108864.0 + b + 0.5) / 4503599627370496.0;
}

// The first `count` N(0, 1) draws of a stream, through `put(k, z)`.
template <typename Put>
void gaussian_stream(uint64_t seed, uint32_t stream, uint64_t count, Put put) {
  const double two_pi = 6.283185307179586;   // nearest double to 2 pi
  for (uint64_t p = 0; 2 * p < count; ++p) {
    const Philox4 r = philox4x32_10(p, stream, seed);
    const double u1 = uniform_from_words(r.w[0], r.w[1]);
    const double u2 = uniform_from_words(r.w[2], r.w[3]);
    const double rad = std::sqrt(-2.0 * std::log(u1));
    put(2 * p, rad * std::cos(two_pi * u2));
    if (2 * p + 1 < count) put(2 * p + 1, rad * std::sin(two_pi * u2));
  }
}

}  // namespace

namespace tq {
bool on_handle_device(const tq_rotation* h) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  return dev == h->device;
}
}  // namespace tq

extern "C" {

const char* tq_status_string(int status) {
  switch (status) {
    case TQ_OK: return "ok";
    case TQ_EINVAL: return "invalid argument";
    case TQ_EUNSUPPORTED: return "unsupported configuration";
    case TQ_EWORKSPACE: return "workspace missing or too small";
    case TQ_ECUDA: return "CUDA runtime error";
    case TQ_ENOMEM: return "device allocation failed";
    default: return "unknown status";
  }
}

int tq_version(void) { return 100; }

int tq_lloyd_max(int d, int bits, double* levels, double* thresholds) {
  if (d < 3 || d > 65536 || bits < 1 || bits > 8 || !levels || !thresholds) return TQ_EINVAL;
  std::vector<double> lv, th;
  if (!lloyd_max_levels(d, bits, &lv, &th)) return TQ_EINVAL;
  std::memcpy(levels, lv.data(), lv.size() * sizeof(double));
  std::memcpy(thresholds, th.data(), th.size() * sizeof(double));
  return TQ_OK;
}

int tq_build_rotation_ex(int d, int code_bits, int kind, int residual, const int8_t* signs,
                         const double* gauss_pi, const float* gauss_s, int m, double rope_base,
                         int64_t rope_max_pos, tq_rotation** out) {
  if (!out) return TQ_EINVAL;
  *out = nullptr;
  if (residual != TQ_RES_QJL && residual != TQ_RES_SIGN) return TQ_EINVAL;
  if (code_bits < 1 || code_bits > 3 || m != d || (residual == TQ_RES_QJL && !gauss_s)) return TQ_EINVAL;
  if (kind == TQ_ROT_HADAMARD) {
    if (!signs) return TQ_EINVAL;
    if (d != 64 && d != 128) return TQ_EUNSUPPORTED;
    for (int i = 0; i < d; ++i)
      if (signs[i] != 1 && signs[i] != -1) return TQ_EINVAL;
  } else if (kind == TQ_ROT_DENSE) {
    if (!gauss_pi) return TQ_EINVAL;
    if (d < 32 || d > 4096 || d % 32) return TQ_EUNSUPPORTED;
  } else {
    return TQ_EINVAL;
  }
  if (rope_base < 0.0 || !std::isfinite(rope_base)) return TQ_EINVAL;
  if (rope_base > 0.0 && (rope_max_pos < 1 || rope_max_pos > (int64_t(1) << 31))) return TQ_EINVAL;

  tq_rotation* h = new (std::nothrow) tq_rotation();
  if (!h) return TQ_ENOMEM;
  if (cudaGetDevice(&h->device) != cudaSuccess) { delete h; return TQ_ECUDA; }
  h->d = d;
  h->m = m;
  h->bits = code_bits;
  h->kind = kind;
  h->residual = residual;
  // QJL: E[sign(s.r) s] = sqrt(2/pi) r/||r|| for Gaussian rows s, hence the
  // sqrt(pi/2)/m estimator; the sign correction adds e_bar sign(r) as it is.
  h->res_const = residual == TQ_RES_QJL ? kQjlConst / m : 1.0;
  h->rope_base = rope_base;
  h->rope_max_pos = rope_base > 0.0 ? rope_max_pos : 0;

  if (!lloyd_max_levels(d, code_bits, &h->levels, &h->thresholds)) { release(h); return TQ_EINVAL; }
  {
    unsigned subsets[4];
    h->n_planes = plane_subsets(code_bits, subsets);
    const int n = 1 << code_bits;
    for (int p = 0; p < h->n_planes; ++p) {
      double acc = 0.0;
      for (int idx = 0; idx < n; ++idx) {
        double prod = 1.0;
        for (int k = 0; k < code_bits; ++k)
          if (subsets[p] >> k & 1u) prod *= ((idx >> k) & 1) ? 1.0 : -1.0;
        acc += h->levels[idx] * prod;
      }
      h->walsh[p] = acc / n;
    }
  }

  int st = TQ_OK;
  {
    std::vector<float> lv(h->levels.begin(), h->levels.end());
    std::vector<float> th(h->thresholds.begin(), h->thresholds.end());
    if ((st = upload(&h->d_levels, lv.data(), lv.size())) != TQ_OK) { release(h); return st; }
    if ((st = upload(&h->d_thresholds, th.data(), th.size())) != TQ_OK) { release(h); return st; }
  }
  if (kind == TQ_ROT_HADAMARD) {
    std::vector<float> sg(d);
    for (int i = 0; i < d; ++i) sg[i] = static_cast<float>(signs[i]);
    if ((st = upload(&h->d_signs, sg.data(), sg.size())) != TQ_OK) { release(h); return st; }
    h->signs = sg;
  } else {
    std::vector<double> pi;
    haar_from_gaussian(gauss_pi, d, &pi);
    std::vector<float> pf(pi.begin(), pi.end());
    if ((st = upload(&h->d_pi, pf.data(), pf.size())) != TQ_OK) { release(h); return st; }
    // bf16 hi + lo pieces of Pi (each rounded to nearest)
    std::vector<uint16_t> ph(pf.size()), pl(pf.size());
    for (size_t i = 0; i < pf.size(); ++i) {
      const float hv = round_to_bf16(pf[i]);
      const float lv = round_to_bf16(pf[i] - hv);
      uint32_t hb, lb;
      std::memcpy(&hb, &hv, 4);
      std::memcpy(&lb, &lv, 4);
      ph[i] = static_cast<uint16_t>(hb >> 16);
      pl[i] = static_cast<uint16_t>(lb >> 16);
    }
    if ((st = upload(&h->d_pi_hi, ph.data(), ph.size())) != TQ_OK) { release(h); return st; }
    if ((st = upload(&h->d_pi_lo, pl.data(), pl.size())) != TQ_OK) { release(h); return st; }
  }
  {
    std::vector<float> s(static_cast<size_t>(m) * d), stt(static_cast<size_t>(d) * m);
    for (int j = 0; j < m; ++j)
      for (int i = 0; i < d; ++i) {
        // the sign correction keeps the residual's own coordinates: S = I
        const float v = residual == TQ_RES_SIGN ? (i == j ? 1.f : 0.f)
                                                : round_to_bf16(gauss_s[static_cast<size_t>(j) * d + i]);
        s[static_cast<size_t>(j) * d + i] = v;
        stt[static_cast<size_t>(i) * m + j] = v;
      }
    if ((st = upload(&h->d_s, s.data(), s.size())) != TQ_OK) { release(h); return st; }
    if ((st = upload(&h->d_st, stt.data(), stt.size())) != TQ_OK) { release(h); return st; }
    if (kind == TQ_ROT_DENSE) {
      std::vector<uint16_t> sb(s.size());
      for (size_t i = 0; i < s.size(); ++i) {
        uint32_t bits;
        std::memcpy(&bits, &s[i], 4);
        sb[i] = static_cast<uint16_t>(bits >> 16);   // S is bf16-exact
      }
      if ((st = upload(&h->d_s_bf16, sb.data(), sb.size())) != TQ_OK) { release(h); return st; }
    }
    if (kind == TQ_ROT_HADAMARD) {
      // K-major bf16 operand with a 128-byte swizzle: K/64 blocks of m rows x
      // 64 elements; row r of a block at (r/8)*1024 + (r%8)*128 bytes, its
      // 16-byte chunk c stored at chunk position c ^ (r%8).  S is
      // bf16-exact, so the upper half of each float is the bf16 value.
      std::vector<uint16_t> op(static_cast<size_t>(m) * d);
      for (int j = 0; j < m; ++j)
        for (int k = 0; k < d; ++k) {
          const size_t off = static_cast<size_t>(k >> 6) * (static_cast<size_t>(m) * 128) + (j >> 3) * 1024 +
                             (j & 7) * 128 + ((((k & 63) >> 3) ^ (j & 7)) << 4) + ((k & 7) << 1);
          uint32_t bits;
          std::memcpy(&bits, &s[static_cast<size_t>(j) * d + k], 4);
          op[off / 2] = static_cast<uint16_t>(bits >> 16);
        }
      if ((st = upload(&h->d_s_op, op.data(), op.size())) != TQ_OK) { release(h); return st; }
      if (d == 128 || d == 64) {
        // H D with H[j][k] = (-1)^popcount(j & k): rows j (output coordinate),
        // K = k, entries +-1 exact in fp16 (0x3C00) and bf16 (0x3F80)
        std::vector<uint16_t> hf(static_cast<size_t>(d) * d), hb(static_cast<size_t>(d) * d);
        for (int j = 0; j < d; ++j)
          for (int k = 0; k < d; ++k) {
            const size_t off = static_cast<size_t>(k >> 6) * (static_cast<size_t>(d) * 128) + (j >> 3) * 1024 +
                               (j & 7) * 128 + ((((k & 63) >> 3) ^ (j & 7)) << 4) + ((k & 7) << 1);
            const bool neg = (__builtin_popcount(static_cast<unsigned>(j & k)) & 1) != (h->signs[k] < 0.f);
            hf[off / 2] = neg ? 0xBC00u : 0x3C00u;
            hb[off / 2] = neg ? 0xBF80u : 0x3F80u;
          }
        if ((st = upload(&h->d_hd_f16, hf.data(), hf.size())) != TQ_OK) { release(h); return st; }
        if ((st = upload(&h->d_hd_bf16, hb.data(), hb.size())) != TQ_OK) { release(h); return st; }
      }
      if (d == 64 && m == 64) {
        // output transform of the tensor-core encoder attention (see
        // tq_internal.h): three [64 x 64] bf16 operands, rows i = output
        // coordinate, K = slot k standing for coordinate dim(k)
        auto slot_dim = [](int k) { return 32 * (k >> 5) + ((k >> 1) & 15) + 16 * (k & 1); };
        auto had = [](int i, int j) { return (__builtin_popcount(static_cast<unsigned>(i & j)) & 1) ? -1.0 : 1.0; };
        const double qjl = h->res_const;
        std::vector<uint16_t> ep(static_cast<size_t>(3) * d * d);
        for (int i = 0; i < d; ++i)
          for (int k = 0; k < d; ++k) {
            const int dk = slot_dim(k);
            const double sgn = h->signs[i] < 0.f ? -1.0 : 1.0;
            double g = 0.0;   // sum_t H[i][t] S[dk][t]
            for (int t = 0; t < d; ++t) g += had(i, t) * s[static_cast<size_t>(dk) * d + t];
            const float b1 = static_cast<float>(sgn * had(i, dk) / 8.0);
            const float b2 = static_cast<float>(sgn * qjl * g / 8.0);
            const float b2h = round_to_bf16(b2), b2l = round_to_bf16(b2 - b2h);
            const size_t off = static_cast<size_t>((i >> 3) * 1024 + (i & 7) * 128 + ((((k >> 3) ^ (i & 7))) << 4) +
                                                   ((k & 7) << 1)) / 2;
            const float vals[3] = {b1, b2h, b2l};
            for (int t = 0; t < 3; ++t) {
              uint32_t bits;
              std::memcpy(&bits, &vals[t], 4);
              ep[static_cast<size_t>(t) * d * d + off] = static_cast<uint16_t>(bits >> 16);
            }
          }
        if ((st = upload(&h->d_enc_epi, ep.data(), ep.size())) != TQ_OK) { release(h); return st; }
      }
    }
  }
  if (rope_base > 0.0) {
    const int half = d / 2;
    h->rope_hi_rows = static_cast<int>((rope_max_pos + kRopeLoRows - 1) / kRopeLoRows);
    std::vector<double> theta(half);
    for (int i = 0; i < half; ++i) theta[i] = std::pow(rope_base, -2.0 * i / d);
    for (int i = 0; i < half && i < 64; ++i) {
      h->rope_th_hi[i] = static_cast<float>(theta[i]);
      h->rope_th_lo[i] = static_cast<float>(theta[i] - static_cast<double>(h->rope_th_hi[i]));
    }
    std::vector<float2> hi(static_cast<size_t>(h->rope_hi_rows) * half), lo(static_cast<size_t>(kRopeLoRows) * half);
    for (int r = 0; r < h->rope_hi_rows; ++r)
      for (int i = 0; i < half; ++i) {
        const double a = static_cast<double>(r) * kRopeLoRows * theta[i];
        hi[static_cast<size_t>(r) * half + i] = make_float2(static_cast<float>(std::cos(a)), static_cast<float>(std::sin(a)));
      }
    for (int r = 0; r < kRopeLoRows; ++r)
      for (int i = 0; i < half; ++i) {
        const double a = static_cast<double>(r) * theta[i];
        lo[static_cast<size_t>(r) * half + i] = make_float2(static_cast<float>(std::cos(a)), static_cast<float>(std::sin(a)));
      }
    if ((st = upload(&h->d_rope_hi, hi.data(), hi.size())) != TQ_OK) { release(h); return st; }
    if ((st = upload(&h->d_rope_lo, lo.data(), lo.size())) != TQ_OK) { release(h); return st; }
  }
  *out = h;
  return TQ_OK;
}

int tq_rotation_draws(int d, int kind, uint64_t seed, int m, int8_t* signs, double* gauss_pi, float* gauss_s) {
  if (d < 1 || d > 4096 || m < 1 || m > 4096) return TQ_EINVAL;
  if (kind != TQ_ROT_HADAMARD && kind != TQ_ROT_DENSE) return TQ_EINVAL;
  if (signs) {
    for (int i = 0; i < d; ++i) signs[i] = (philox4x32_10(static_cast<uint64_t>(i), kStreamSigns, seed).w[0] >> 31) ? -1 : 1;
  }
  if (gauss_s) {
    gaussian_stream(seed, kStreamQjl, static_cast<uint64_t>(m) * d,
                    [&](uint64_t k, double z) { gauss_s[k] = static_cast<float>(z); });
  }
  if (gauss_pi && kind == TQ_ROT_DENSE) {
    gaussian_stream(seed, kStreamDense, static_cast<uint64_t>(d) * d, [&](uint64_t k, double z) { gauss_pi[k] = z; });
  }
  return TQ_OK;
}

int tq_build_rotation(int d, int code_bits, int kind, const int8_t* signs, const double* gauss_pi,
                      const float* gauss_s, int m, double rope_base, int64_t rope_max_pos, tq_rotation** out) {
  return tq_build_rotation_ex(d, code_bits, kind, TQ_RES_QJL, signs, gauss_pi, gauss_s, m, rope_base, rope_max_pos,
                              out);
}

int tq_build_rotation_seeded(int d, int code_bits, int kind, int residual, uint64_t seed, int m, double rope_base,
                             int64_t rope_max_pos, tq_rotation** out) {
  if (!out) return TQ_EINVAL;
  *out = nullptr;
  if (d < 1 || d > 4096 || m != d) return TQ_EINVAL;
  if (kind != TQ_ROT_HADAMARD && kind != TQ_ROT_DENSE) return TQ_EINVAL;
  std::vector<int8_t> sg(d);
  std::vector<float> gs(static_cast<size_t>(m) * d);
  std::vector<double> gp(kind == TQ_ROT_DENSE ? static_cast<size_t>(d) * d : 0);
  const int st = tq_rotation_draws(d, kind, seed, m, sg.data(), gp.empty() ? nullptr : gp.data(), gs.data());
  if (st != TQ_OK) return st;
  return tq_build_rotation_ex(d, code_bits, kind, residual, sg.data(), gp.empty() ? nullptr : gp.data(), gs.data(), m,
                              rope_base, rope_max_pos, out);
}

int tq_free_rotation(tq_rotation* h) {
  release(h);
  return TQ_OK;
}

int tq_rotation_dims(const tq_rotation* h, int* d, int* m, int* bits, int64_t* code_bytes,
                     int64_t* sign_bytes) {
  if (!h) return TQ_EINVAL;
  if (d) *d = h->d;
  if (m) *m = h->m;
  if (bits) *bits = h->bits;
  if (code_bytes) *code_bytes = static_cast<int64_t>(h->bits) * h->d / 8;
  if (sign_bytes) *sign_bytes = h->m / 8;
  return TQ_OK;
}

int tq_rotation_export(const tq_rotation* h, float* pi, float* s, double* levels, double* thresholds) {
  if (!h) return TQ_EINVAL;
  const int d = h->d, m = h->m;
  if (pi) {
    if (h->kind == TQ_ROT_DENSE) {
      if (cudaMemcpy(pi, h->d_pi, sizeof(float) * d * d, cudaMemcpyDeviceToHost) != cudaSuccess) return TQ_ECUDA;
    } else {
      std::vector<float> sg(d);
      if (cudaMemcpy(sg.data(), h->d_signs, sizeof(float) * d, cudaMemcpyDeviceToHost) != cudaSuccess) return TQ_ECUDA;
      const float inv = 1.0f / std::sqrt(static_cast<float>(d));
      for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) {
          const int par = __builtin_popcount(static_cast<unsigned>(i & j)) & 1;
          pi[static_cast<size_t>(i) * d + j] = (par ? -1.0f : 1.0f) * sg[j] * inv;
        }
    }
  }
  if (s && cudaMemcpy(s, h->d_s, sizeof(float) * m * d, cudaMemcpyDeviceToHost) != cudaSuccess) return TQ_ECUDA;
  if (levels) std::memcpy(levels, h->levels.data(), h->levels.size() * sizeof(double));
  if (thresholds) std::memcpy(thresholds, h->thresholds.data(), h->thresholds.size() * sizeof(double));
  return TQ_OK;
}

}  // extern "C"
