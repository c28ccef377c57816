// Normalize-Shift-Normalize record mode ([NSNQuant] §1 and §4): the per-block
// shift that turns a block of tokens into the vectors the codec encodes.
//
// For one block (a sequence and head) of L tokens x_t, after RoPE at
// positions pos_offset + t when the handle has RoPE ([TurboESM] §2.A):
//   s1_t = ||x~_t|| / sqrt(d),  o = mean_t x~_t / s1_t  (per channel),
//   x'_t = x~_t - s1_t o.
// x'_t is NSN's s1 s2 x3: the same direction as the twice-normalised token,
// with norm s1 s2 sqrt(d).  The codec then encodes x' (no RoPE) into an
// ordinary record; s1 per token and o per block stay beside the record, and
// decode adds s1_t <q', o> to the score and o sum_t p_t s1_t to the output.
// Three launches: chunk sums of x~ / s1 (enough chunks to fill the GPU),
// their mean per block, and x' for every row.
#include <cuda_bf16.h>

#include "tq_internal.h"

namespace {

constexpr int kNsnWarps = 8;

// Row t of block blk after RoPE, lane l holding coordinates l + 32 j (the
// RoPE pairs (i, i + d/2) meet in the lane); returns s1 = ||x~|| / sqrt(d).
template <int D, typename T>
__device__ __forceinline__ float nsn_row(const T* __restrict__ x, int64_t blk, int64_t L, int64_t ld, int64_t t,
                                         int64_t pos_offset, int rope, const float2* __restrict__ rope_hi,
                                         const float2* __restrict__ rope_lo, int lane, float (&v)[D / 32]) {
  constexpr int J = D / 32;
  const T* row = x + (blk * L + t) * ld;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    if constexpr (sizeof(T) == 4) v[j] = row[lane + 32 * j];
    else v[j] = __bfloat162float(row[lane + 32 * j]);
  }
  if (rope) {
    const int64_t pos = pos_offset + t;
#pragma unroll
    for (int j = 0; j < J / 2; ++j) {
      const int i = lane + 32 * j;   // pair (i, i + D/2)
      const float2 a = rope_hi[(pos >> kRopeLoBits) * (D / 2) + i];
      const float2 b = rope_lo[(pos & (kRopeLoRows - 1)) * (D / 2) + i];
      const float cs = a.x * b.x - a.y * b.y, sn = a.y * b.x + a.x * b.y;
      const float x1 = v[j], x2 = v[j + J / 2];
      v[j] = x1 * cs - x2 * sn;
      v[j + J / 2] = x2 * cs + x1 * sn;
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < J; ++j) ss = fmaf(v[j], v[j], ss);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, s);
  return sqrtf(ss) * rsqrtf(static_cast<float>(D));
}

// 1. Per (block, chunk): the sum over the chunk's rows of x~ / s1 (zero rows
// add zero), in double, warps in a fixed order: part[blk][chunk][D]; with one
// chunk per block, o itself (part unused).
template <int D, typename T>
__global__ void __launch_bounds__(kNsnWarps * 32) nsn_sum_kernel(const T* __restrict__ x, int64_t L, int64_t ld,
                                                                int64_t chunk, int64_t pos_offset, int rope,
                                                                const float2* __restrict__ rope_hi,
                                                                const float2* __restrict__ rope_lo,
                                                                double* __restrict__ part, float* __restrict__ o) {
  constexpr int J = D / 32;
  __shared__ double wsum[kNsnWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t blk = blockIdx.y, c = blockIdx.x;
  const int64_t t_end = min(L, (c + 1) * chunk);
  double acc[J];
#pragma unroll
  for (int j = 0; j < J; ++j) acc[j] = 0.0;
  for (int64_t t = c * chunk + warp; t < t_end; t += kNsnWarps) {
    float v[J];
    const float s1 = nsn_row<D, T>(x, blk, L, ld, t, pos_offset, rope, rope_hi, rope_lo, lane, v);
    const float inv = s1 > 0.f ? 1.f / s1 : 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j) acc[j] += static_cast<double>(v[j] * inv);
  }
#pragma unroll
  for (int j = 0; j < J; ++j) wsum[warp][lane + 32 * j] = acc[j];
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < kNsnWarps; ++w) s += wsum[w][i];
    if (gridDim.x == 1) o[blk * D + i] = L > 0 ? static_cast<float>(s / static_cast<double>(L)) : 0.f;
    else part[(blk * gridDim.x + c) * D + i] = s;
  }
}

// 2. o of each block: the chunk sums in order, over L.
template <int D>
__global__ void nsn_mean_kernel(const double* __restrict__ part, int n_chunks, int64_t L, float* __restrict__ o) {
  const int64_t blk = blockIdx.x;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    double s = 0.0;
    for (int c = 0; c < n_chunks; ++c) s += part[(blk * n_chunks + c) * D + i];
    o[blk * D + i] = L > 0 ? static_cast<float>(s / static_cast<double>(L)) : 0.f;
  }
}

// 3. x' = x~ - s1 o for every row (one warp per row, grid-stride).
template <int D, typename T>
__global__ void __launch_bounds__(kNsnWarps * 32) nsn_apply_kernel(const T* __restrict__ x, int64_t n_blocks, int64_t L,
                                                                  int64_t ld, int64_t pos_offset, int rope,
                                                                  const float2* __restrict__ rope_hi,
                                                                  const float2* __restrict__ rope_lo,
                                                                  const float* __restrict__ o,
                                                                  float* __restrict__ x_shift,
                                                                  float* __restrict__ s1_out) {
  constexpr int J = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t n = n_blocks * L;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kNsnWarps;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * kNsnWarps + (threadIdx.x >> 5); r < n; r += stride) {
    const int64_t blk = r / L, t = r - blk * L;
    float v[J];
    const float s1 = nsn_row<D, T>(x, blk, L, ld, t, pos_offset, rope, rope_hi, rope_lo, lane, v);
    float* dst = x_shift + r * D;
#pragma unroll
    for (int j = 0; j < J; ++j) dst[lane + 32 * j] = fmaf(-s1, o[blk * D + lane + 32 * j], v[j]);
    if (lane == 0) s1_out[r] = s1;
  }
}

template <int D, typename T>
int launch_nsn(const tq_rotation* h, const void* x, int64_t n_blocks, int64_t L, int64_t ld, int64_t pos_offset,
               int rope, float* x_shift, float* s1, float* o, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // chunks of at least 256 rows, about 4 CTAs per SM over all blocks
  int64_t n_chunks = (4 * static_cast<int64_t>(sms) + n_blocks - 1) / n_blocks;
  const int64_t max_chunks = (L + 255) / 256;
  if (n_chunks > max_chunks) n_chunks = max_chunks;
  if (n_chunks < 1) n_chunks = 1;
  if (n_chunks > 65535) n_chunks = 65535;
  const int64_t chunk = L > 0 ? (L + n_chunks - 1) / n_chunks : 1;
  // with two or more chunks (then L > 256 and n_chunks <= L / 2) the chunk
  // sums ([n_blocks][n_chunks][D] doubles, at most half of x_shift) live in
  // x_shift until the last kernel overwrites it; one chunk writes o directly
  double* part = reinterpret_cast<double*>(x_shift);
  const T* xp = static_cast<const T*>(x);
  nsn_sum_kernel<D, T><<<dim3(static_cast<unsigned>(n_chunks), static_cast<unsigned>(n_blocks)), kNsnWarps * 32, 0, s>>>(
      xp, L, ld, chunk, pos_offset, rope, h->d_rope_hi, h->d_rope_lo, part, o);
  if (n_chunks > 1)
    nsn_mean_kernel<D><<<static_cast<unsigned>(n_blocks), D, 0, s>>>(part, static_cast<int>(n_chunks), L, o);
  const int64_t rows = n_blocks * L;
  const int64_t want = (rows + kNsnWarps - 1) / kNsnWarps;
  const int64_t cap = 8 * static_cast<int64_t>(sms);
  const unsigned grid = static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap));
  nsn_apply_kernel<D, T><<<grid, kNsnWarps * 32, 0, s>>>(xp, n_blocks, L, ld, pos_offset, rope, h->d_rope_hi,
                                                        h->d_rope_lo, o, x_shift, s1);
  return tq::launch_status();
}

}  // namespace

extern "C" int tq_nsn_shift(const tq_rotation* h, const void* x, int dtype, int64_t n_blocks, int64_t L, int64_t ld,
                            int64_t pos_offset, int apply_rope, float* x_shift, float* s1, float* o, void* stream) {
  if (!h || n_blocks < 0 || L < 0 || (dtype != TQ_F32 && dtype != TQ_BF16)) return TQ_EINVAL;
  if (n_blocks == 0) return TQ_OK;
  if (n_blocks > 65535) return TQ_EUNSUPPORTED;   // one grid row of the sum kernel per block
  if (!x || !x_shift || !s1 || !o || ld < h->d) return TQ_EINVAL;
  if (reinterpret_cast<uintptr_t>(x_shift) & 7u) return TQ_EINVAL;   // holds double partial sums first
  if (h->d != 64 && h->d != 128) return TQ_EUNSUPPORTED;
  if (apply_rope) {
    if (h->rope_base <= 0.0 || pos_offset < 0) return TQ_EINVAL;
    if (L > 0 && pos_offset + L - 1 >= h->rope_max_pos) return TQ_EINVAL;
  }
  if (!tq::on_handle_device(h)) return TQ_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rope = apply_rope ? 1 : 0;
  if (h->d == 128)
    return dtype == TQ_F32 ? launch_nsn<128, float>(h, x, n_blocks, L, ld, pos_offset, rope, x_shift, s1, o, s)
                           : launch_nsn<128, __nv_bfloat16>(h, x, n_blocks, L, ld, pos_offset, rope, x_shift, s1, o, s);
  return dtype == TQ_F32 ? launch_nsn<64, float>(h, x, n_blocks, L, ld, pos_offset, rope, x_shift, s1, o, s)
                         : launch_nsn<64, __nv_bfloat16>(h, x, n_blocks, L, ld, pos_offset, rope, x_shift, s1, o, s);
}
