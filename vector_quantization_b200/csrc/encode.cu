// Encode kernel: RoPE -> norm -> randomized Hadamard rotation -> Lloyd-Max
// codes -> residual -> QJL sign sketch -> bit-packed record.
//
// [TurboESM] §2.A (RoPE before the rotation), §2.D (residual x - x_hat),
// §3 (quantization and packing paid at prefill); [TurboQuant] "Principe",
// Étape 1 (rotation, per-coordinate quantizer, norm kept) and Étape 2 /
// "QJL" (one sign bit per Johnson-Lindenstrauss projection of the residual);
// [NSNQuant] §2 (randomized Hadamard transform, H D / sqrt(d)).
//
// Layout inside a warp: lane l holds coordinates l + 32 j (j < D/32).  Bits
// 0..4 of a coordinate index are then the lane id and bits 5.. the register
// index, so the fast Walsh-Hadamard transform needs 5 shuffle stages plus
// log2(D/32) in-register stages, and a warp ballot over one register yields
// one 32-bit word of a bit-plane (coordinates 32 j .. 32 j + 31) directly.
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
  const float* dsigns;  // [D]
  const float* st;      // [D][D] S transposed (st[i*D + j] = S[j][i])
  const float* thresholds;
  const float* levels;
  const float2* rope_hi;
  const float2* rope_lo;
  int64_t rope_max_pos;
};

template <typename T>
__device__ __forceinline__ float load_elem(const T* p);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

template <int D, int BITS, typename T>
__global__ void __launch_bounds__(256) encode_hadamard_kernel(EncodeParams p) {
  constexpr int NJ = D / 32;
  constexpr int NT = (1 << BITS) - 1;
  extern __shared__ float smem[];
  float* st = smem;                                       // [D][D]
  float* rbuf = smem + D * D + (threadIdx.x >> 5) * D;    // per-warp residual
  __shared__ float thr_s[NT];
  __shared__ float lev_s[1 << BITS];

  for (int i = threadIdx.x; i < D * D; i += blockDim.x) st[i] = p.st[i];
  if (threadIdx.x < NT) thr_s[threadIdx.x] = p.thresholds[threadIdx.x];
  if (threadIdx.x < (1 << BITS)) lev_s[threadIdx.x] = p.levels[threadIdx.x];
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * warps + (threadIdx.x >> 5);
  const int64_t step = static_cast<int64_t>(gridDim.x) * warps;
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  float dsg[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) dsg[j] = p.dsigns[lane + 32 * j];

  for (int64_t row = first; row < p.n; row += step) {
    const T* xr = static_cast<const T*>(p.x) + row * p.ld;
    float v[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) v[j] = load_elem<T>(xr + lane + 32 * j);

    const int64_t rec = row * p.out_stride;
    if (p.rope) {
      const int64_t pos = p.pos ? p.pos[row] : p.pos_offset + row % p.pos_period;
      if (pos < 0 || pos >= p.rope_max_pos) {
        if (lane == 0) p.norms[rec] = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
        continue;
      }
      const float2* hi = p.rope_hi + (pos >> kRopeLoBits) * (D / 2);
      const float2* lo = p.rope_lo + (pos & (kRopeLoRows - 1)) * (D / 2);
#pragma unroll
      for (int j = 0; j < NJ / 2; ++j) {
        const int i = lane + 32 * j;
        const float2 a = hi[i], b = lo[i];
        // cos/sin of (hi + lo) angle by angle addition
        const float c = a.x * b.x - a.y * b.y;
        const float s = a.y * b.x + a.x * b.y;
        const float x1 = v[j], x2 = v[j + NJ / 2];
        v[j] = x1 * c - x2 * s;
        v[j + NJ / 2] = x2 * c + x1 * s;
      }
    }

    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) ss = fmaf(v[j], v[j], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float norm = sqrtf(ss);
    const float inv = norm > 0.f ? 1.0f / norm : 0.f;

    // u = D x / ||x||, then y = H u / sqrt(d) (Sylvester order)
    float u[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) u[j] = v[j] * inv * dsg[j];
#pragma unroll
    for (int s = 0; s < 5; ++s) {
      const bool upper = (lane >> s) & 1;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const float o = __shfl_xor_sync(0xffffffffu, u[j], 1 << s);
        u[j] = upper ? o - u[j] : u[j] + o;
      }
    }
#pragma unroll
    for (int b = 1; b < NJ; b <<= 1) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        if (j & b) continue;
        const float a0 = u[j], a1 = u[j | b];
        u[j] = a0 + a1;
        u[j | b] = a0 - a1;
      }
    }

    int idx[NJ];
    float r[NJ];
    float rr = 0.f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const float y = u[j] * inv_sqrt_d;
      int c = 0;
#pragma unroll
      for (int t = 0; t < NT; ++t) c += (y >= thr_s[t]) ? 1 : 0;
      idx[j] = c;
      r[j] = norm * (y - lev_s[c]);
      rr = fmaf(r[j], r[j], rr);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rr += __shfl_xor_sync(0xffffffffu, rr, o);

    uint32_t* crec = p.codes + rec * (BITS * NJ);
#pragma unroll
    for (int k = 0; k < BITS; ++k) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const uint32_t w = __ballot_sync(0xffffffffu, (idx[j] >> k) & 1);
        if (lane == k * NJ + j) crec[k * NJ + j] = w;
      }
    }

    // QJL: (S r)_jr for jr = lane + 32 jj; S^T in shared memory.
#pragma unroll
    for (int j = 0; j < NJ; ++j) rbuf[lane + 32 * j] = r[j];
    __syncwarp();
    float acc[NJ];
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) acc[jj] = 0.f;
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
      const float ri = rbuf[i];
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) acc[jj] = fmaf(st[i * D + lane + 32 * jj], ri, acc[jj]);
    }
    __syncwarp();
    uint32_t* srec = p.signs + rec * NJ;
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) {
      const uint32_t w = __ballot_sync(0xffffffffu, acc[jj] >= 0.f);
      if (lane == jj) srec[jj] = w;
    }
    if (lane == 0) p.norms[rec] = make_float2(norm, sqrtf(rr));
  }
}

template <int D, int BITS, typename T>
int launch_encode(const EncodeParams& p, cudaStream_t stream) {
  const int threads = 256;
  const size_t smem = sizeof(float) * (D * D + (threads / 32) * D);
  auto kern = encode_hadamard_kernel<D, BITS, T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return TQ_ECUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (p.n + threads / 32 - 1) / (threads / 32);
  const int blocks = static_cast<int>(need < sms * 4LL ? need : sms * 4LL);
  kern<<<blocks, threads, smem, stream>>>(p);
  return tq::launch_status();
}

template <int D, typename T>
int dispatch_bits(int bits, const EncodeParams& p, cudaStream_t s) {
  switch (bits) {
    case 1: return launch_encode<D, 1, T>(p, s);
    case 2: return launch_encode<D, 2, T>(p, s);
    case 3: return launch_encode<D, 3, T>(p, s);
  }
  return TQ_EUNSUPPORTED;
}

}  // namespace

extern "C" int tq_quantize_kv(const tq_rotation* h, const void* x, int dtype, int64_t n, int64_t ld,
                              const int64_t* pos, int64_t pos_period, int64_t pos_offset,
                              int apply_rope, uint8_t* codes, uint8_t* signs, float* norms,
                              int64_t out_stride, void* stream) {
  if (!h) return TQ_EINVAL;
  if (n < 0 || (dtype != TQ_F32 && dtype != TQ_BF16)) return TQ_EINVAL;
  if (n == 0) return TQ_OK;
  if (!x || !codes || !signs || !norms || out_stride < 1 || ld < h->d) return TQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(signs) & 3u) ||
      (reinterpret_cast<uintptr_t>(norms) & 7u))
    return TQ_EINVAL;
  if (dtype == TQ_F32 ? (ld % 4 != 0 || !tq::aligned16(x)) : (ld % 8 != 0 || !tq::aligned16(x))) return TQ_EINVAL;
  if (apply_rope) {
    if (h->rope_base <= 0.0) return TQ_EINVAL;
    if (!pos) {
      if (pos_period < 1 || pos_offset < 0) return TQ_EINVAL;
      const int64_t hi = pos_offset + (n < pos_period ? n : pos_period) - 1;
      if (hi >= h->rope_max_pos) return TQ_EINVAL;
    }
  }
  if (h->kind != TQ_ROT_HADAMARD) return TQ_EUNSUPPORTED;
  if (!tq::on_handle_device(h)) return TQ_EINVAL;

  EncodeParams p{};
  p.x = x;
  p.n = n;
  p.ld = ld;
  p.pos = pos;
  p.pos_period = pos_period < 1 ? 1 : pos_period;
  p.pos_offset = pos_offset;
  p.rope = apply_rope ? 1 : 0;
  p.codes = reinterpret_cast<uint32_t*>(codes);
  p.signs = reinterpret_cast<uint32_t*>(signs);
  p.norms = reinterpret_cast<float2*>(norms);
  p.out_stride = out_stride;
  p.dsigns = h->d_signs;
  p.st = h->d_st;
  p.thresholds = h->d_thresholds;
  p.levels = h->d_levels;
  p.rope_hi = h->d_rope_hi;
  p.rope_lo = h->d_rope_lo;
  p.rope_max_pos = h->rope_max_pos;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (h->d == 128)
    return dtype == TQ_F32 ? dispatch_bits<128, float>(h->bits, p, s) : dispatch_bits<128, __nv_bfloat16>(h->bits, p, s);
  if (h->d == 64)
    return dtype == TQ_F32 ? dispatch_bits<64, float>(h->bits, p, s) : dispatch_bits<64, __nv_bfloat16>(h->bits, p, s);
  return TQ_EUNSUPPORTED;
}
