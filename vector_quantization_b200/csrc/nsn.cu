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
#include <cuda_bf16.h>

#include "tq_internal.h"

namespace {

constexpr int kNsnWarps = 8;

// One CTA of 8 warps per block; lane l of a warp holds coordinates l + 32 j
// of one row, so the RoPE pairs (i, i + d/2) meet in the lane.
template <int D, typename T>
__global__ void __launch_bounds__(kNsnWarps * 32) nsn_shift_kernel(const T* __restrict__ x, int64_t L, int64_t ld,
                                                                  int64_t pos_offset, int rope,
                                                                  const float2* __restrict__ rope_hi,
                                                                  const float2* __restrict__ rope_lo,
                                                                  float* __restrict__ x_shift,
                                                                  float* __restrict__ s1_out,
                                                                  float* __restrict__ o_out) {
  constexpr int J = D / 32;
  __shared__ double part[kNsnWarps][D];
  __shared__ float o_s[D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t blk = blockIdx.x;
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  // row t of the block after RoPE, and its s1
  auto load = [&](int64_t t, float (&v)[J]) {
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
    return sqrtf(ss) * inv_sqrt_d;
  };
  // pass 1: o = mean of x~ / s1 (zero rows add zero); sums in double (a
  // block holds up to millions of tokens), per warp in a fixed order, then
  // the warps in order
  double acc[J];
#pragma unroll
  for (int j = 0; j < J; ++j) acc[j] = 0.0;
  for (int64_t t = warp; t < L; t += kNsnWarps) {
    float v[J];
    const float s1 = load(t, v);
    const float inv = s1 > 0.f ? 1.f / s1 : 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j) acc[j] += static_cast<double>(v[j] * inv);
  }
#pragma unroll
  for (int j = 0; j < J; ++j) part[warp][lane + 32 * j] = acc[j];
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < kNsnWarps; ++w) s += part[w][i];
    const float o = L > 0 ? static_cast<float>(s / static_cast<double>(L)) : 0.f;
    o_s[i] = o;
    o_out[blk * D + i] = o;
  }
  __syncthreads();
  // pass 2: x' = x~ - s1 o
  for (int64_t t = warp; t < L; t += kNsnWarps) {
    float v[J];
    const float s1 = load(t, v);
    float* dst = x_shift + (blk * L + t) * D;
#pragma unroll
    for (int j = 0; j < J; ++j) dst[lane + 32 * j] = fmaf(-s1, o_s[lane + 32 * j], v[j]);
    if (lane == 0) s1_out[blk * L + t] = s1;
  }
}

template <int D, typename T>
int launch_nsn(const tq_rotation* h, const void* x, int64_t n_blocks, int64_t L, int64_t ld, int64_t pos_offset,
               int rope, float* x_shift, float* s1, float* o, cudaStream_t s) {
  nsn_shift_kernel<D, T><<<static_cast<unsigned>(n_blocks), kNsnWarps * 32, 0, s>>>(
      static_cast<const T*>(x), L, ld, pos_offset, rope, h->d_rope_hi, h->d_rope_lo, x_shift, s1, o);
  return tq::launch_status();
}

}  // namespace

extern "C" int tq_nsn_shift(const tq_rotation* h, const void* x, int dtype, int64_t n_blocks, int64_t L, int64_t ld,
                            int64_t pos_offset, int apply_rope, float* x_shift, float* s1, float* o, void* stream) {
  if (!h || n_blocks < 0 || L < 0 || (dtype != TQ_F32 && dtype != TQ_BF16)) return TQ_EINVAL;
  if (n_blocks == 0) return TQ_OK;
  if (n_blocks > 0x7fffffff) return TQ_EUNSUPPORTED;
  if (!x || !x_shift || !s1 || !o || ld < h->d) return TQ_EINVAL;
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
