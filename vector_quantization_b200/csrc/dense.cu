// Encoding with a dense rotation (any d that is a multiple of 32; used where
// d is not a power of two, e.g. d = 1536 for vector search).
//
// [TurboQuant] "Principe", Étape 1: random rotation, then a scalar Lloyd-Max
// quantizer per coordinate with the vector norm kept; Étape 2 / "QJL": sign
// bits of the Johnson-Lindenstrauss projection of the residual plus ||r||.
// With a dense rotation both y = Pi x and S r are genuine dense
// contractions; they run on the tensor core (tc_gemm.cu) over a chunk of
// vectors, with fp32 operands split into bf16 hi + lo pieces:
//   1. X -> X_hi, X_lo (bf16)
//   2. Y = X Pi^T          (X_hi Pi_hi + X_hi Pi_lo + X_lo Pi_hi, fp32 accumulate)
//   3. per row: ||x||, y = Y / ||x||, codes (bit-planes by warp ballot),
//      r = ||x|| (y - c[idx]) written as bf16 hi + lo over X_hi, X_lo, ||r||
//   4. P = R S^T           (R_hi S + R_lo S; S is bf16-exact)
//   5. per row: sign bits of P by warp ballot
// The split keeps each product within ~2^-16 relative, so rotated unit
// coordinates stay ~1e-7 from the exact values (sum of d products of random
// sign), far inside the 1e-5 boundary band that decides code parity.
#include <cuda_bf16.h>

#include <cmath>

#include "tq_internal.h"

namespace {

constexpr int kBM = 128, kBN = 128, kBK = 8;

// C[M][N] = A[M][K] * B[N][K]^T (all row-major), fp32.
__global__ void __launch_bounds__(256) sgemm_nt_kernel(int M, int N, int K, const float* __restrict__ A, int64_t lda,
                                                        const float* __restrict__ B, int64_t ldb, float* __restrict__ C,
                                                        int64_t ldc) {
  __shared__ __align__(16) float As[kBK][kBM + 4];
  __shared__ __align__(16) float Bs[kBK][kBN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  // loader: row lr = tid / 2, k-offset lk = (tid & 1) * 4 of both tiles
  const int lr = tid >> 1, lk = (tid & 1) * 4;
  for (int k0 = 0; k0 < K; k0 += kBK) {
    {
      const int gm = m0 + lr, gk = k0 + lk;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (gm < M) {
        const float* src = A + gm * lda + gk;
        if (gk + 3 < K) v = *reinterpret_cast<const float4*>(src);
        else {
          v.x = gk < K ? src[0] : 0.f;
          v.y = gk + 1 < K ? src[1] : 0.f;
          v.z = gk + 2 < K ? src[2] : 0.f;
        }
      }
      As[lk + 0][lr] = v.x;
      As[lk + 1][lr] = v.y;
      As[lk + 2][lr] = v.z;
      As[lk + 3][lr] = v.w;
    }
    {
      const int gn = n0 + lr, gk = k0 + lk;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (gn < N) {
        const float* src = B + gn * ldb + gk;
        if (gk + 3 < K) v = *reinterpret_cast<const float4*>(src);
        else {
          v.x = gk < K ? src[0] : 0.f;
          v.y = gk + 1 < K ? src[1] : 0.f;
          v.z = gk + 2 < K ? src[2] : 0.f;
        }
      }
      Bs[lk + 0][lr] = v.x;
      Bs[lk + 1][lr] = v.y;
      Bs[lk + 2][lr] = v.z;
      Bs[lk + 3][lr] = v.w;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kBK; ++k) {
      float a[8], b[8];
      const float4 a0 = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[k][64 + tx * 4]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w; a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w; b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (gn < N) C[gm * ldc + gn] = acc[i][j];
    }
  }
}

// One warp per row: norms, codes (bit-planes), residual written over Y.
template <int BITS>
__global__ void __launch_bounds__(256) dense_quantize_rows_kernel(const float* __restrict__ x, int64_t ld, int64_t n,
                                                                  int d, const float* __restrict__ yr,
                                                                  __nv_bfloat16* __restrict__ rh,
                                                                  __nv_bfloat16* __restrict__ rl,
                                                                  const float* __restrict__ thresholds,
                                                                  const float* __restrict__ levels,
                                                                  uint32_t* __restrict__ codes, float2* __restrict__ norms,
                                                                  int sign_res) {
  constexpr int NT = (1 << BITS) - 1;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n) return;
  float thr[NT], lev[1 << BITS];
#pragma unroll
  for (int t = 0; t < NT; ++t) thr[t] = thresholds[t];
#pragma unroll
  for (int t = 0; t < (1 << BITS); ++t) lev[t] = levels[t];
  const float* xr = x + row * ld;
  float ss = 0.f;
  for (int i = lane; i < d; i += 32) ss = fmaf(xr[i], xr[i], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float norm = sqrtf(ss);
  const float inv = norm > 0.f ? 1.0f / norm : 0.f;
  const float* y = yr + row * d;
  const int words = d / 32;
  uint32_t* crec = codes + row * (BITS * words);
  float rr = 0.f;
  for (int w = 0; w < words; ++w) {
    const float yv = y[32 * w + lane] * inv;
    int c = 0;
#pragma unroll
    for (int t = 0; t < NT; ++t) c += (yv >= thr[t]) ? 1 : 0;
    const float r = norm * (yv - lev[c]);
    const __nv_bfloat16 h = __float2bfloat16_rn(r);
    rh[row * d + 32 * w + lane] = h;
    rl[row * d + 32 * w + lane] = __float2bfloat16_rn(r - __bfloat162float(h));
    rr = sign_res ? rr + fabsf(r) : fmaf(r, r, rr);   // sign-residual handles keep mean |r_i|
#pragma unroll
    for (int k = 0; k < BITS; ++k) {
      const uint32_t bits = __ballot_sync(0xffffffffu, (c >> k) & 1);
      if (lane == k) crec[k * words + w] = bits;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) rr += __shfl_xor_sync(0xffffffffu, rr, o);
  if (lane == 0) norms[row] = make_float2(norm, sign_res ? rr / static_cast<float>(d) : sqrtf(rr));
}

// One warp per row: sign bits of P = R S^T.
__global__ void __launch_bounds__(256) dense_sign_rows_kernel(const float* __restrict__ proj, int64_t n, int m,
                                                              uint32_t* __restrict__ signs) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n) return;
  const float* pr = proj + row * m;
  const int words = m / 32;
  for (int w = 0; w < words; ++w) {
    const uint32_t bits = __ballot_sync(0xffffffffu, pr[32 * w + lane] >= 0.f);
    if (lane == 0) signs[row * words + w] = bits;
  }
}

}  // namespace

namespace tq {

int sgemm_nt(int M, int N, int K, const float* A, int64_t lda, const float* B, int64_t ldb, float* C, int64_t ldc,
             cudaStream_t s) {
  if (M <= 0 || N <= 0) return TQ_OK;
  dim3 grid((N + kBN - 1) / kBN, (M + kBM - 1) / kBM);
  sgemm_nt_kernel<<<grid, 256, 0, s>>>(M, N, K, A, lda, B, ldb, C, ldc);
  return launch_status();
}

// Bytes of dense-encode scratch per vector of a chunk: X (then R) as bf16
// hi + lo, and Y (then P) as fp32 (m = d).
size_t dense_bytes_per_row(const tq_rotation* h) { return static_cast<size_t>(h->d) * 4 + static_cast<size_t>(h->m) * 4; }

}  // namespace tq

extern "C" size_t tq_quantize_dense_workspace_size(const tq_rotation* h, int64_t n) {
  if (!h || n < 0) return 0;
  const int64_t chunk = n < 32768 ? (n < 1 ? 1 : n) : 32768;
  return static_cast<size_t>(chunk) * tq::dense_bytes_per_row(h);
}

extern "C" int tq_quantize_dense(const tq_rotation* h, const float* x, int64_t n, int64_t ld, uint8_t* codes,
                                 uint8_t* signs, float* norms, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!h || n < 0) return TQ_EINVAL;
  if (n == 0) return TQ_OK;
  if (h->kind != TQ_ROT_DENSE) return TQ_EUNSUPPORTED;
  if (!x || !codes || !signs || !norms || ld < h->d || (ld & 3) || !tq::aligned16(x)) return TQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(signs) & 3u) ||
      (reinterpret_cast<uintptr_t>(norms) & 7u))
    return TQ_EINVAL;
  const size_t per_row = tq::dense_bytes_per_row(h);
  if (!workspace || workspace_bytes < per_row || !tq::aligned16(workspace)) return TQ_EWORKSPACE;
  if (!tq::on_handle_device(h)) return TQ_EINVAL;
  const int d = h->d, m = h->m;
  const int64_t chunk = static_cast<int64_t>(workspace_bytes / per_row);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t cbytes = static_cast<int64_t>(h->bits) * d / 8, sbytes = m / 8;
  for (int64_t r0 = 0; r0 < n; r0 += chunk) {
    const int64_t rows = n - r0 < chunk ? n - r0 : chunk;
    // scratch of the chunk: X (later R) as bf16 hi, lo; Y (later P) as fp32
    uint16_t* xh = static_cast<uint16_t*>(workspace);
    uint16_t* xl = xh + rows * d;
    float* yr = reinterpret_cast<float*>(xl + rows * d);
    int st = tq::split_bf16(x + r0 * ld, ld, rows, d, xh, xl, d, s);
    if (st != TQ_OK) return st;
    if ((st = tq::tc_gemm_split(static_cast<int>(rows), d, d, xh, xl, d, h->d_pi_hi, h->d_pi_lo, d, yr, d, s)) != TQ_OK)
      return st;
    const int blocks = static_cast<int>((rows + 7) / 8);
    uint32_t* cw = reinterpret_cast<uint32_t*>(codes + r0 * cbytes);
    float2* nw = reinterpret_cast<float2*>(norms) + r0;
    __nv_bfloat16* rh = reinterpret_cast<__nv_bfloat16*>(xh);
    __nv_bfloat16* rl = reinterpret_cast<__nv_bfloat16*>(xl);
    const int sres = h->residual == TQ_RES_SIGN ? 1 : 0;
    switch (h->bits) {
      case 1: dense_quantize_rows_kernel<1><<<blocks, 256, 0, s>>>(x + r0 * ld, ld, rows, d, yr, rh, rl, h->d_thresholds, h->d_levels, cw, nw, sres); break;
      case 2: dense_quantize_rows_kernel<2><<<blocks, 256, 0, s>>>(x + r0 * ld, ld, rows, d, yr, rh, rl, h->d_thresholds, h->d_levels, cw, nw, sres); break;
      default: dense_quantize_rows_kernel<3><<<blocks, 256, 0, s>>>(x + r0 * ld, ld, rows, d, yr, rh, rl, h->d_thresholds, h->d_levels, cw, nw, sres); break;
    }
    if ((st = tq::launch_status()) != TQ_OK) return st;
    if ((st = tq::tc_gemm_split(static_cast<int>(rows), m, d, xh, xl, d, h->d_s_bf16, nullptr, d, yr, m, s)) != TQ_OK)
      return st;
    dense_sign_rows_kernel<<<blocks, 256, 0, s>>>(yr, rows, m, reinterpret_cast<uint32_t*>(signs + r0 * sbytes));
    if ((st = tq::launch_status()) != TQ_OK) return st;
  }
  return TQ_OK;
}
