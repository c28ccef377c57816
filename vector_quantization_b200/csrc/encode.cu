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
// bit-plane directly.  A warp works on two vectors at a time as independent
// chains; RoPE takes cos/sin of each row's position from the two-level tables
// (angle addition of a coarse and a fine angle).  The QJL projection S r of
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
constexpr int kEncWarps = kEncThreads / 32;
constexpr int kWaitLimit = 1 << 22;

template <int D, int BITS, typename T>
__global__ void __launch_bounds__(kEncThreads) encode_hadamard_kernel(EncodeParams p) {
  constexpr int NJ = D / 32;
  constexpr int NT = (1 << BITS) - 1;
  constexpr int OPB = kTileVec * D * 2;           // bytes of one bf16 [128 x D] operand
  constexpr int SB = D * D * 2;                   // bytes of S [m x d] bf16
  const int R = p.rows;                           // vectors per tile
  const int RUN = R >= kEncWarps ? R / kEncWarps : 1;   // vectors per warp per tile (contiguous run)
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
  float thr[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) thr[t] = thr_s[t];
  uint32_t phase = 0;
  const int64_t n_tiles = (p.n + R - 1) / R;

  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t row0 = tile * R;
    bool ok = true;
    // ---------------- per-vector work: warp owns a run of RUN vectors ---------
    // Two vectors per step as independent chains, so their shuffle and
    // load latencies overlap.  The Walsh-Hadamard transform runs on the
    // unnormalised vector (it is linear), so the norm reduction overlaps it.
    int64_t pos_base = 0;   // position of the run's first row when pos == NULL
    if (p.rope && !p.pos) {
      const int64_t r0w = row0 + static_cast<int64_t>(warp) * RUN;
      pos_base = r0w < p.n ? r0w % p.pos_period : 0;
    }
    for (int q0 = 0; q0 < RUN; q0 += 2) {
      float x[2][NJ];
      bool valid[2], pos_ok[2];
      int64_t row[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int q = q0 + c;
        const int vl = warp * RUN + q;
        row[c] = row0 + vl;
        valid[c] = q < RUN && vl < R && row[c] < p.n;
        pos_ok[c] = true;
        const T* xr = static_cast<const T*>(p.x) + (valid[c] ? row[c] : 0) * p.ld;
#pragma unroll
        for (int j = 0; j < NJ; ++j) x[c][j] = load_elem<T>(xr + lane + 32 * j);
      }
      if (p.rope) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          int64_t pos;
          if (p.pos) {
            pos = valid[c] ? p.pos[row[c]] : 0;
          } else {
            int64_t m = pos_base + q0 + c;
            if (m >= p.pos_period) m %= p.pos_period;
            pos = p.pos_offset + m;
          }
          pos_ok[c] = pos >= 0 && pos < p.rope_max_pos;
          const int64_t pc = pos_ok[c] ? pos : 0;
          // cos/sin(pos theta_i) from the two-level tables (angle addition)
          const float2* hi = p.rope_hi + (pc >> kRopeLoBits) * (D / 2);
          const float2* lo = p.rope_lo + (pc & (kRopeLoRows - 1)) * (D / 2);
#pragma unroll
          for (int j = 0; j < NJ / 2; ++j) {
            const float2 a = hi[lane + 32 * j], b = lo[lane + 32 * j];
            const float cs = a.x * b.x - a.y * b.y, sn = a.y * b.x + a.x * b.y;
            const float x1 = x[c][j], x2 = x[c][j + NJ / 2];
            x[c][j] = x1 * cs - x2 * sn;
            x[c][j + NJ / 2] = x2 * cs + x1 * sn;
          }
        }
      }
      // u = H D x (unnormalised, Sylvester order); lane l holds u[l + 32 j]
      float u[2][NJ], ss[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        ss[c] = 0.f;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          ss[c] = fmaf(x[c][j], x[c][j], ss[c]);
          u[c][j] = x[c][j] * dsg[j];
        }
      }
#pragma unroll
      for (int st = 0; st < 5; ++st) {
        const bool upper = (lane >> st) & 1;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, u[c][j], 1 << st);
            u[c][j] = upper ? o - u[c][j] : u[c][j] + o;
          }
          ss[c] += __shfl_xor_sync(0xffffffffu, ss[c], 16 >> st);
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int bb = 1; bb < NJ; bb <<= 1)
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            if (j & bb) continue;
            const float a0 = u[c][j], a1 = u[c][j | bb];
            u[c][j] = a0 + a1;
            u[c][j | bb] = a0 - a1;
          }
      float r[2][NJ], rr[2], nrm[2];
      int idx[2][NJ];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        nrm[c] = sqrtf(ss[c]);
        const float scale = (nrm[c] > 0.f ? 1.0f / nrm[c] : 0.f) * inv_sqrt_d;
        const bool keep = valid[c] && pos_ok[c];
        rr[c] = 0.f;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const float y = u[c][j] * scale;   // coordinate of the unit vector
          int ci = 0;
#pragma unroll
          for (int t = 0; t < NT; ++t) ci += (y >= thr[t]) ? 1 : 0;
          idx[c][j] = ci;
          r[c][j] = keep ? nrm[c] * (y - lev_s[ci]) : 0.f;
          rr[c] = fmaf(r[c][j], r[c][j], rr[c]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int c = 0; c < 2; ++c) rr[c] += __shfl_xor_sync(0xffffffffu, rr[c], o);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (q0 + c >= RUN || warp * RUN + q0 + c >= R) break;
        if (valid[c]) {
          const int64_t rec = row[c] * p.out_stride;
          if (pos_ok[c]) {
            uint32_t* crec = p.codes + rec * (BITS * NJ);
#pragma unroll
            for (int k = 0; k < BITS; ++k) {
#pragma unroll
              for (int j = 0; j < NJ; ++j) {
                const uint32_t w = __ballot_sync(0xffffffffu, (idx[c][j] >> k) & 1);
                if (lane == k * NJ + j) crec[k * NJ + j] = w;
              }
            }
            if (lane == 0) p.norms[rec] = make_float2(nrm[c], sqrtf(rr[c]));
          } else if (lane == 0) {
            p.norms[rec] = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
          }
        }
        // residual as two bf16 pieces, row v of the A operand of S r
        const int v = warp * RUN + q0 + c;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const __nv_bfloat16 h = __float2bfloat16_rn(r[c][j]);
          const __nv_bfloat16 l = __float2bfloat16_rn(r[c][j] - __bfloat162float(h));
          const uint32_t off = tqtc::sw128_offset(v, lane + 32 * j, kTileVec);
          *reinterpret_cast<__nv_bfloat16*>(r_hi + off) = h;
          *reinterpret_cast<__nv_bfloat16*>(r_lo + off) = l;
        }
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
    ok = tqtc::mbar_wait(&mbar, phase, kWaitLimit) && ok;
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
