// Encode kernel: RoPE -> norm -> randomized Hadamard rotation -> Lloyd-Max
// codes -> residual -> QJL sign sketch -> bit-packed record.
//
// [TurboESM] §2.A (RoPE before the rotation), §2.D (residual x - x_hat),
// §3 (quantization and packing paid at prefill); [TurboQuant] "Principe",
// Étape 1 (rotation, per-coordinate quantizer, norm kept) and Étape 2 /
// "QJL" (one sign bit per Johnson-Lindenstrauss projection of the residual);
// [NSNQuant] §2 (randomized Hadamard transform, H D / sqrt(d)).
//
// A CTA encodes tiles of R vectors (R = 8..128, chosen per call so that
// small batches still spread over many SMs).  Per-vector work runs one warp per
// vector: lane l holds coordinates l + 32 j (j < D/32), so the fast
// Walsh-Hadamard transform needs 5 shuffle stages plus log2(D/32) in-register
// stages, and a warp ballot over one register yields one 32-bit word of a
// bit-plane directly.  Each warp takes a run of consecutive rows, so RoPE
// advances its cos/sin by one position with an angle-addition step and reads
// the two-level tables only where positions jump.  The QJL projection S r of
// the whole tile is a dense product and runs on the 5th-generation tensor
// core (tcgen05, M = 128 rows; rows past R stay zero): r is written as bf16
// hi/lo pieces into a 128-byte swizzled shared-memory operand, S (bf16-exact,
// stored by the handle already in operand layout) stays resident in shared
// memory, the fp32 result lands in tensor memory and each thread reads back
// its vector's row to form the sign bits.
#include <cuda_bf16.h>

#include "bitplane.cuh"
#include "tcgen05.cuh"
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
  const uint16_t* s_op; // S, bf16 bits in the swizzled K-major operand layout
  int rows;             // vectors per tile, R in {8, 16, 32, 64, 128}
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

// Tile of 128 vectors per CTA iteration (the M of one tensor-core product).
constexpr int kTileVec = 128;
constexpr int kEncThreads = 256;
constexpr int kWaitLimit = 1 << 22;

template <int D, int BITS, typename T>
__global__ void __launch_bounds__(kEncThreads) encode_hadamard_kernel(EncodeParams p) {
  constexpr int NJ = D / 32;
  constexpr int NT = (1 << BITS) - 1;
  constexpr int OPB = kTileVec * D * 2;           // bytes of one bf16 [128 x D] operand
  constexpr int SB = D * D * 2;                   // bytes of S [m x d] bf16
  const int R = p.rows;                           // vectors per tile
  const int RUN = R / (kEncThreads / 32);         // vectors per warp per tile (contiguous run)
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t mbar;
  __shared__ uint32_t tmem_slot;
  __shared__ float thr_s[NT];
  __shared__ float lev_s[1 << BITS];
  uint8_t* base = raw + ((1024 - (tqtc::smem_u32(raw) & 1023)) & 1023);
  uint8_t* s_op = base;               // S, K-major SW128 (rows j = sketch index, k = coordinate)
  uint8_t* r_hi = base + SB;          // residual tile, hi bf16 piece
  uint8_t* r_lo = base + SB + OPB;    // residual tile, lo bf16 piece

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int c = tid; c < SB / 16; c += blockDim.x) tqdev::cp_async16(s_op + 16 * c, p.s_op + 8 * c, 16);
  tqdev::cp_async_commit();
  if (R < kTileVec) {
    // rows R..127 of the residual operand are never written: keep them zero
    for (int c = tid; c < 2 * OPB / 16; c += blockDim.x) reinterpret_cast<uint4*>(r_hi)[c] = make_uint4(0, 0, 0, 0);
  }
  if (tid < NT) thr_s[tid] = p.thresholds[tid];
  if (tid < (1 << BITS)) lev_s[tid] = p.levels[tid];
  if (tid == 0) tqtc::mbar_init(&mbar, 1);
  if (warp == 0) tqtc::tmem_alloc(&tmem_slot, D < 32 ? 32 : D);
  tqdev::cp_async_wait<0>();
  tqtc::fence_before_sync();
  __syncthreads();
  tqtc::fence_after_sync();
  const uint32_t tmem = tmem_slot;
  const uint32_t idesc = tqtc::idesc_bf16_f32(kTileVec, D);
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  float dsg[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) dsg[j] = p.dsigns[lane + 32 * j];
  // rotation by one position of the frequencies this lane owns (i = lane + 32 j, j < NJ/2)
  float2 step[NJ / 2 > 0 ? NJ / 2 : 1];
  if (p.rope) {
#pragma unroll
    for (int j = 0; j < NJ / 2; ++j) step[j] = p.rope_lo[(D / 2) + lane + 32 * j];
  }
  uint32_t phase = 0;
  const int64_t n_tiles = (p.n + R - 1) / R;

  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t row0 = tile * R;
    // ---------------- per-vector work: warp owns a run of RUN vectors ---------
    float2 cs[NJ / 2 > 0 ? NJ / 2 : 1];
    int64_t prev_pos = -2;
    for (int q = 0; q < RUN; ++q) {
      const int v = warp * RUN + q;
      const int64_t row = row0 + v;
      float r[NJ];
      bool valid = row < p.n;
      if (valid) {
        const T* xr = static_cast<const T*>(p.x) + row * p.ld;
        float x[NJ];
#pragma unroll
        for (int j = 0; j < NJ; ++j) x[j] = load_elem<T>(xr + lane + 32 * j);
        const int64_t rec = row * p.out_stride;
        if (p.rope) {
          const int64_t pos = p.pos ? p.pos[row] : p.pos_offset + row % p.pos_period;
          if (pos < 0 || pos >= p.rope_max_pos) {
            if (lane == 0) p.norms[rec] = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
            valid = false;
          } else {
            if (pos != prev_pos + 1) {
              // seed cos/sin(pos theta_i) from the two-level tables (angle addition)
              const float2* hi = p.rope_hi + (pos >> kRopeLoBits) * (D / 2);
              const float2* lo = p.rope_lo + (pos & (kRopeLoRows - 1)) * (D / 2);
#pragma unroll
              for (int j = 0; j < NJ / 2; ++j) {
                const float2 a = hi[lane + 32 * j], b = lo[lane + 32 * j];
                cs[j] = make_float2(a.x * b.x - a.y * b.y, a.y * b.x + a.x * b.y);
              }
            } else {
              // advance one position: (c, s) <- rotation by theta_i
#pragma unroll
              for (int j = 0; j < NJ / 2; ++j)
                cs[j] = make_float2(cs[j].x * step[j].x - cs[j].y * step[j].y, cs[j].y * step[j].x + cs[j].x * step[j].y);
            }
            prev_pos = pos;
#pragma unroll
            for (int j = 0; j < NJ / 2; ++j) {
              const float x1 = x[j], x2 = x[j + NJ / 2];
              x[j] = x1 * cs[j].x - x2 * cs[j].y;
              x[j + NJ / 2] = x2 * cs[j].x + x1 * cs[j].y;
            }
          }
        }
        if (valid) {
          float ss = 0.f;
#pragma unroll
          for (int j = 0; j < NJ; ++j) ss = fmaf(x[j], x[j], ss);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          const float norm = sqrtf(ss);
          const float inv = norm > 0.f ? 1.0f / norm : 0.f;
          // y = H (D x / ||x||) / sqrt(d), Sylvester order; lane l holds y[l + 32 j]
          float u[NJ];
#pragma unroll
          for (int j = 0; j < NJ; ++j) u[j] = x[j] * inv * dsg[j];
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
          if (lane == 0) p.norms[rec] = make_float2(norm, sqrtf(rr));
        }
      }
      if (!valid) {
#pragma unroll
        for (int j = 0; j < NJ; ++j) r[j] = 0.f;
      }
      // residual as two bf16 pieces, row v of the A operand of S r
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const __nv_bfloat16 h = __float2bfloat16_rn(r[j]);
        const __nv_bfloat16 l = __float2bfloat16_rn(r[j] - __bfloat162float(h));
        const uint32_t off = tqtc::sw128_offset(v, lane + 32 * j, kTileVec);
        *reinterpret_cast<__nv_bfloat16*>(r_hi + off) = h;
        *reinterpret_cast<__nv_bfloat16*>(r_lo + off) = l;
      }
    }
    // ---------------- S r on the tensor core: D[v][j] = sum_k R[v][k] S[j][k] --
    tqtc::fence_smem_to_async();
    tqtc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      tqtc::fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tqtc::mma_bf16_ss(tmem, tqtc::sw128_desc_kstep(tqtc::smem_u32(r_hi), ks, kTileVec),
                          tqtc::sw128_desc_kstep(tqtc::smem_u32(s_op), ks, D), idesc, ks > 0);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tqtc::mma_bf16_ss(tmem, tqtc::sw128_desc_kstep(tqtc::smem_u32(r_lo), ks, kTileVec),
                          tqtc::sw128_desc_kstep(tqtc::smem_u32(s_op), ks, D), idesc, true);
      tqtc::mma_commit(&mbar);
    }
    const bool ok = tqtc::mbar_wait(&mbar, phase, kWaitLimit);
    phase ^= 1;
    tqtc::fence_after_sync();
    // ---------------- sign bits: warp w reads lanes 32 (w % 4).., half the columns
    {
      const int quad = warp & 3, half = warp >> 2;
      const int v = quad * 32 + lane;
      const int64_t row = v < R ? row0 + v : p.n;
      constexpr int COLS = D / 2;
      uint32_t words[COLS / 32];
#pragma unroll
      for (int c = 0; c < COLS / 32; ++c) {
        float val[32];
        tqtc::tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + half * COLS + 32 * c, val);
        uint32_t w = 0;
#pragma unroll
        for (int b = 0; b < 32; ++b) w |= (val[b] >= 0.f ? 1u : 0u) << b;
        words[c] = w;
      }
      if (row < p.n) {
        uint32_t* srec = p.signs + row * p.out_stride * NJ + half * (COLS / 32);
#pragma unroll
        for (int c = 0; c < COLS / 32; ++c) srec[c] = ok ? words[c] : 0u;
        if (!ok && half == 0)
          p.norms[row * p.out_stride] = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
      }
    }
    tqtc::fence_before_sync();
    __syncthreads();
  }
  if (warp == 0) tqtc::tmem_free(tmem, D < 32 ? 32 : D);
}

template <int D, int BITS, typename T>
int launch_encode(const EncodeParams& p, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(D) * D * 2 + 2 * static_cast<size_t>(kTileVec) * D * 2 + 1024;
  auto kern = encode_hadamard_kernel<D, BITS, T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return TQ_ECUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // smallest tile (>= 8 rows, one per warp) that still gives each CTA slot work
  int rows = 8;
  while (rows < kTileVec && (p.n + rows - 1) / rows > 2LL * sms) rows *= 2;
  EncodeParams q = p;
  q.rows = rows;
  const int64_t tiles = (p.n + rows - 1) / rows;
  const int blocks = static_cast<int>(tiles < sms * 2LL ? tiles : sms * 2LL);
  kern<<<blocks, kEncThreads, smem, stream>>>(q);
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
  p.s_op = h->d_s_op;
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
