// Encode parameters and the one-vector encode shared by the encode kernels
// and the decode step's fused append.
//
// [TurboESM] §2.A (RoPE before the rotation), §2.D (residual x - x_hat);
// [TurboQuant] Étape 1 (rotation, per-coordinate quantizer, norm kept) and
// "QJL" (one sign bit per projection of the residual); [NSNQuant] §2
// (randomized Hadamard transform, H D / sqrt(d)).
#pragma once

#include <cuda_bf16.h>

#include "tq_internal.h"

namespace {

struct EncodeParams {
  const void* x;
  int64_t n, ld;
  const int64_t* pos;
  int64_t pos_period, pos_offset;
  int rope;
  uint32_t* codes;      // record = BITS * D / 32 words
  uint32_t* signs;      // record = D / 32 words (m == D)
  float2* norms;        // record = (||x||, ||r||)
  int64_t out_stride;
  const int64_t* out_rows;  // [n] record of each row (scatter calls), or null: row * out_stride
  int64_t n_records;        // records in the output arrays (scatter calls: targets outside are skipped)
  int sign_res;             // sign-residual handle: norms[1] = mean |r_i| instead of ||r|| (S is the identity)
  float* nsn_s1;            // one-vector encode with an NSN shift: s1 of each record (indexed as the norms)
  const float* dsigns;  // [D]
  const uint16_t* s_op; // S, bf16 bits in the swizzled K-major operand layout
  const uint16_t* hd_op; // tensor-core encode: H D in the same layout (fp16 bits when split, else bf16)
  const float* st;      // S transposed, fp32: st[k * d + j] = S[j][k]
  int rows;             // warp-per-vector kernel: vectors per tile, R in {8, 16, ..., 128}
  const float* thresholds;
  const float* levels;
  const float2* rope_hi;
  const float2* rope_lo;
  int64_t rope_max_pos;
  // thread-per-vector kernel: sign diagonal and the positive half of the
  // (symmetric) codebook, read straight from the parameter space
  float dsg[128];
  float tpos[4];        // thresholds above 0, ascending (2^(b-1) - 1 of them)
  float lpos[4];        // levels above 0, ascending (2^(b-1) of them)
  float2 theta[64];     // tensor-core encode: RoPE frequency i as (hi, lo) float pieces
};

// Output record of input row `row`: row * out_stride, or the row's entry of
// out_rows for scatter calls (-1, not written, when that entry lies outside
// the output arrays).
__device__ __forceinline__ int64_t out_record(const EncodeParams& p, int64_t row) {
  if (!p.out_rows) return row * p.out_stride;
  const int64_t r = p.out_rows[row];
  return r >= 0 && r < p.n_records ? r : -1;
}

// The fields of p that come from the handle: codebook halves, sign
// diagonal, S, RoPE tables and frequencies, residual mode.
inline void fill_handle_fields(EncodeParams& p, const tq_rotation* h) {
  p.sign_res = h->residual == TQ_RES_SIGN ? 1 : 0;
  p.dsigns = h->d_signs;
  p.s_op = h->d_s_op;
  p.st = h->d_st;
  const int half = 1 << (h->bits - 1);
  for (int i = 0; i < h->d && i < 128; ++i) p.dsg[i] = h->signs[i];
  for (int k = 0; k < 4; ++k) {
    p.lpos[k] = k < half ? static_cast<float>(h->levels[half + k]) : 0.f;
    p.tpos[k] = k < half - 1 ? static_cast<float>(h->thresholds[half + k]) : 0.f;
  }
  p.thresholds = h->d_thresholds;
  p.levels = h->d_levels;
  p.rope_hi = h->d_rope_hi;
  p.rope_lo = h->d_rope_lo;
  p.rope_max_pos = h->rope_max_pos;
  for (int i = 0; i < 64; ++i) p.theta[i] = make_float2(h->rope_th_hi[i], h->rope_th_lo[i]);
}

// One vector encoded by a group of D threads, thread i holding coordinate i:
// RoPE pairs meet through shared memory, the norm and ||r|| are group
// reductions, the Walsh-Hadamard transform takes five shuffle stages and
// log2(d/32) shared-memory stages, a warp ballot yields a plane word, and
// (S r)_i is a matrix-vector product on the CUDA cores.
//   xr     the input row; rec its record (>= 0); pos its RoPE position
//   buf    D floats of the group's shared memory, red 2 x D/32 floats
//   sync   the group's barrier; scol(k) = S[i][k]
//   nsn_o  null, or the shift o [D] of the NSN block the row is appended to
//          ([NSNQuant] §1, §4): after RoPE, s1 = ||x~|| / sqrt(d) goes to
//          p.nsn_s1[rec] and the codec encodes x' = x~ - s1 o
// Every early return depends on the row alone (uniform over the group).
template <int D, int BITS, typename T, typename Sync, typename SCol>
__device__ __forceinline__ void encode_vec_core(const EncodeParams& p, int i, const T* xr, int64_t rec, int64_t pos,
                                                float* buf, float (*red)[D / 32], Sync sync, SCol scol,
                                                const float* nsn_o = nullptr) {
  constexpr int NW = D / 32;
  const int lane = i & 31, w = i >> 5;
  float x;
  if constexpr (sizeof(T) == 4) x = __ldg(reinterpret_cast<const float*>(xr) + i);
  else x = __bfloat162float(xr[i]);
  if (p.rope) {
    if (pos < 0 || pos >= p.rope_max_pos) {
      if (i == 0) p.norms[rec] = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
      return;
    }
    buf[i] = x;
    sync();
    const int j = i & (D / 2 - 1);
    const float2 a = p.rope_hi[(pos >> kRopeLoBits) * (D / 2) + j];
    const float2 b = p.rope_lo[(pos & (kRopeLoRows - 1)) * (D / 2) + j];
    const float cs = a.x * b.x - a.y * b.y, sn = a.y * b.x + a.x * b.y;
    const float x1 = buf[j], x2 = buf[j + D / 2];
    x = i < D / 2 ? x1 * cs - x2 * sn : x2 * cs + x1 * sn;
  }
  if (nsn_o) {
    // s1 from a group reduction (red[1] is free until the residual sums,
    // several barriers later)
    float s = x * x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[1][w] = s;
    sync();
    s = 0.f;
#pragma unroll
    for (int q = 0; q < NW; ++q) s += red[1][q];
    const float s1 = sqrtf(s) * rsqrtf(static_cast<float>(D));
    x = fmaf(-s1, __ldg(nsn_o + i), x);
    if (i == 0) p.nsn_s1[rec] = s1;
  }
  // ||x|| and u = H D x (unnormalised, Sylvester order)
  float ss = x * x;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  float u = x * p.dsg[i];
#pragma unroll
  for (int bit = 1; bit < 32; bit <<= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, u, bit);
    u = (lane & bit) ? o - u : u + o;
  }
  if (lane == 0) red[0][w] = ss;
#pragma unroll
  for (int bit = 32; bit < D; bit <<= 1) {
    sync();
    buf[i] = u;
    sync();
    const float o = buf[i ^ bit];
    u = (i & bit) ? o - u : u + o;
  }
  sync();
  ss = 0.f;
#pragma unroll
  for (int q = 0; q < NW; ++q) ss += red[0][q];
  const float nrm = sqrtf(ss);
  const float y = fmaf(u, (nrm > 0.f ? 1.0f / nrm : 0.f) * rsqrtf(static_cast<float>(D)), 0.f);   // -0 -> +0
  // symmetric codebook: sign picks the half, |y| against the positive thresholds the level
  const bool pos_half = y >= 0.f;
  const float a = fabsf(y);
  uint32_t bits[BITS];
  float mag;
  if constexpr (BITS == 1) {
    bits[0] = pos_half;
    mag = p.lpos[0];
  } else if constexpr (BITS == 2) {
    const bool o = a >= p.tpos[0];
    bits[1] = pos_half;
    bits[0] = pos_half == o;
    mag = o ? p.lpos[1] : p.lpos[0];
  } else {
    const bool m1 = a >= p.tpos[0], m2 = a >= p.tpos[1], m3 = a >= p.tpos[2];
    bits[2] = pos_half;
    bits[1] = pos_half == m2;
    bits[0] = pos_half == (m1 != (m2 != m3));
    mag = m3 ? p.lpos[3] : (m2 ? p.lpos[2] : (m1 ? p.lpos[1] : p.lpos[0]));
  }
  const float r = nrm * (y - copysignf(mag, y));
  uint32_t* crec = p.codes + rec * (BITS * NW);
#pragma unroll
  for (int k = 0; k < BITS; ++k) {
    const uint32_t word = __ballot_sync(0xffffffffu, bits[k]);
    if (lane == 0) crec[k * NW + w] = word;
  }
  float rr = p.sign_res ? fabsf(r) : r * r;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) rr += __shfl_xor_sync(0xffffffffu, rr, o);
  if (lane == 0) red[1][w] = rr;
  buf[i] = r;
  sync();
  // (S r)_i
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int k = 0; k < D; k += 4) {
    const float4 rv = *reinterpret_cast<const float4*>(buf + k);
    acc[0] = fmaf(scol(k), rv.x, acc[0]);
    acc[1] = fmaf(scol(k + 1), rv.y, acc[1]);
    acc[2] = fmaf(scol(k + 2), rv.z, acc[2]);
    acc[3] = fmaf(scol(k + 3), rv.w, acc[3]);
  }
  const float proj = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  const uint32_t sword = __ballot_sync(0xffffffffu, proj >= 0.f);
  if (lane == 0) p.signs[rec * NW + w] = sword;
  if (i == 0) {
    rr = 0.f;
#pragma unroll
    for (int q = 0; q < NW; ++q) rr += red[1][q];
    p.norms[rec] = make_float2(nrm, p.sign_res ? rr * (1.f / D) : sqrtf(rr));
  }
}

}  // namespace
