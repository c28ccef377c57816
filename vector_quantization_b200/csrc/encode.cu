// Encode kernel: RoPE -> norm -> randomized Hadamard rotation -> Lloyd-Max
// codes -> residual -> QJL sign sketch -> bit-packed record.
//
// [TurboESM] §2.A (RoPE before the rotation), §2.D (residual x - x_hat),
// §3 (quantization and packing paid at prefill); [TurboQuant] "Principe",
// Étape 1 (rotation, per-coordinate quantizer, norm kept) and Étape 2 /
// "QJL" (one sign bit per Johnson-Lindenstrauss projection of the residual);
// [NSNQuant] §2 (randomized Hadamard transform, H D / sqrt(d)).
//
// The kernel (encode_rows_kernel, below) gives each thread one whole vector
// in registers; the QJL projection S r of each 128-vector tile is a dense
// product and runs on the 5th-generation tensor core (tcgen05).
#include <cuda_bf16.h>

#include "bitplane.cuh"
#include "encode_vec.cuh"
#include "tcgen05.cuh"
#include "tq_internal.h"

namespace {

// Tile of 128 vectors per CTA iteration (the M of one tensor-core product).
constexpr int kTileVec = 128;
constexpr int kWaitLimit = 1 << 17;   // polls of about 9 us each: a wait gives up after about a second

// ===========================================================================
// Block-per-vector encode, for the few vectors a decode step appends: one
// vector per block of D threads (encode_vec_core), with row i of S loaded
// into registers before the wait on the previous launch, so its loads
// overlap that launch's tail.
// ===========================================================================
template <int D, int BITS, typename T>
__device__ __forceinline__ void encode_vec_body(const EncodeParams& p) {
  __shared__ __align__(16) float buf[D];
  __shared__ float red[2][D / 32];
  const int i = threadIdx.x;
  const int64_t row = blockIdx.x;
  float scol[D];   // row i of S
#pragma unroll
  for (int k = 0; k < D; ++k) scol[k] = __ldg(p.st + k * D + i);
  // S belongs to the handle; everything below may depend on the previous
  // launch on the stream (programmatic dependent launch)
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int64_t rec = out_record(p, row);
  if (rec < 0) return;   // uniform over the block (one vector per block)
  const int64_t pos = p.rope ? (p.pos ? p.pos[row] : p.pos_offset + row % p.pos_period) : 0;
  encode_vec_core<D, BITS, T>(p, i, static_cast<const T*>(p.x) + row * p.ld, rec, pos, buf, red,
                              [] { __syncthreads(); }, [&](int k) { return scol[k]; });
}

template <int D, int BITS, typename T>
__global__ void __launch_bounds__(D) encode_vec_kernel(const __grid_constant__ EncodeParams p) {
  encode_vec_body<D, BITS, T>(p);
}

// The same for two row sets of equal count, d and bits in one launch (the
// keys and values a decode step appends): blockIdx.y picks the set.
template <int D, int BITS, typename T>
__global__ void __launch_bounds__(D) encode_vec_pair_kernel(const __grid_constant__ EncodeParams pk,
                                                           const __grid_constant__ EncodeParams pv) {
  if (blockIdx.y == 0) encode_vec_body<D, BITS, T>(pk);
  else encode_vec_body<D, BITS, T>(pv);
}

// Batches up to this many vectors take the block-per-vector kernel.
constexpr int64_t kVecKernelMaxN = 256;

// ===========================================================================
// Warp-per-vector encode, for small batches (a decode step's new keys and
// values): lane l of a warp holds coordinates l + 32 j, the Walsh-Hadamard
// transform takes 5 shuffle stages plus log2(d/32) in-register stages, and a
// ballot over one register yields a bit-plane word.  Its per-vector latency
// is far below the thread-per-vector kernel's, which wins on throughput.
// ===========================================================================
constexpr int kEncThreads = 256;
constexpr int kEncWarps = kEncThreads / 32;

template <typename T>
__device__ __forceinline__ float load_elem(const T* p);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// Tile of 128 vectors per CTA iteration (the M of one tensor-core product).

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
          rr[c] = p.sign_res ? rr[c] + fabsf(r[c][j]) : fmaf(r[c][j], r[c][j], rr[c]);
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
          const int64_t rec = out_record(p, row[c]);
          if (rec < 0) continue;
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
            if (lane == 0) p.norms[rec] = make_float2(nrm[c], p.sign_res ? rr[c] * (1.f / D) : sqrtf(rr[c]));
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
      const int64_t rec = row < p.n ? out_record(p, row) : -1;
      if (rec >= 0) {
        uint32_t* srec = p.signs + rec * NJ + half * (COLS / 32);
#pragma unroll
        for (int c = 0; c < COLS / 32; ++c) srec[c] = ok ? words[c] : 0u;
        if (!ok && half == 0) p.norms[rec] = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
      }
    }
    tqtc::fence_before_sync();
    __syncthreads();
  }
  if (warp == 0) tqtc::tmem_free(tmem, D < 32 ? 32 : D);
}

template <int D, int BITS, typename T>
int launch_encode_warp(const EncodeParams& p, cudaStream_t stream) {
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

// ===========================================================================
// Thread-per-vector encode.  Each thread holds one whole vector in registers,
// so RoPE, the norm, the Walsh-Hadamard transform (log2 d in-register
// butterfly stages) and the quantizer need no cross-lane traffic, and each
// bit-plane word is assembled in the thread.  A CTA is two groups of four
// warps; a group owns one 128-row tile (thread t = row t = tensor-memory lane
// t), its own residual operand and accumulator, and synchronises with a named
// barrier, so one group's tensor-core product and read-back overlap the other
// group's per-vector work.  S (shared by both groups) is resident in shared
// memory in operand layout.
// ===========================================================================
constexpr int kRowThreads = 256;    // two groups
constexpr int kGroupThreads = 128;  // one tile row per thread

__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(1 + g), "r"(kGroupThreads) : "memory");
}

// Row of D elements (16-byte aligned) into fp32 registers.
template <int D, typename T>
__device__ __forceinline__ void load_row(const T* xr, float (&u)[D]) {
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr) + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        u[8 * c + 2 * q] = __uint_as_float(w[q] << 16);
        u[8 * c + 2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(xr) + c);
      u[4 * c] = v.x;
      u[4 * c + 1] = v.y;
      u[4 * c + 2] = v.z;
      u[4 * c + 3] = v.w;
    }
  }
}

// Unnormalised Sylvester-order Walsh-Hadamard transform in registers.
template <int D>
__device__ __forceinline__ void fwht_regs(float (&u)[D]) {
#pragma unroll
  for (int h = 1; h < D; h <<= 1)
#pragma unroll
    for (int i = 0; i < D; ++i)
      if (!(i & h)) {
        const float a = u[i], b = u[i | h];
        u[i] = a + b;
        u[i | h] = a - b;
      }
}

// Codes of 32 coordinates y[i] (unit-vector coordinates, never -0), as BITS
// plane words, and their residuals norm * (y - level) written over y.  The
// codebook is symmetric: the sign picks the half and |y| against the positive
// thresholds t_k picks the level m within it, idx = pos ? 2^(b-1) + m :
// 2^(b-1) - 1 - m.  Every plane bit is then an XNOR of sign bits: s_y (y < 0)
// and s_k (|y| - t_k < 0, exact in fp32): bit b-1 = !s_y, bit b-2 = s_y == s_1
// (b = 2: s_0), bit 0 (b = 3) = s_y == s_0 ^ s_1 ^ s_2.  Bits are shifted in
// with one funnel shift each and the words complemented at the end.
// nl[k] = norm * lpos[k].  Returns the sum of squared residuals.
template <int BITS>
__device__ __forceinline__ float quantize32(float* y, const float (&tp)[4], const float (&nl)[4], float norm,
                                            uint32_t (&w)[BITS]) {
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] = 0;
  float rr = 0.f;
#pragma unroll
  for (int i = 31; i >= 0; --i) {
    const float v = y[i];
    const uint32_t sy = __float_as_uint(v);
    const float a = fabsf(v);
    float nmag;
    if constexpr (BITS == 1) {
      w[0] = __funnelshift_l(sy, w[0], 1);
      nmag = nl[0];
    } else if constexpr (BITS == 2) {
      const uint32_t s0 = __float_as_uint(a - tp[0]);
      w[1] = __funnelshift_l(sy, w[1], 1);
      w[0] = __funnelshift_l(sy ^ s0, w[0], 1);
      nmag = a >= tp[0] ? nl[1] : nl[0];
    } else {
      const uint32_t s0 = __float_as_uint(a - tp[0]), s1 = __float_as_uint(a - tp[1]),
                     s2 = __float_as_uint(a - tp[2]);
      w[2] = __funnelshift_l(sy, w[2], 1);
      w[1] = __funnelshift_l(sy ^ s1, w[1], 1);
      w[0] = __funnelshift_l(sy ^ s0 ^ s1 ^ s2, w[0], 1);
      nmag = a >= tp[2] ? nl[3] : (a >= tp[1] ? nl[2] : (a >= tp[0] ? nl[1] : nl[0]));
    }
    const float r = fmaf(norm, v, -copysignf(nmag, v));
    y[i] = r;
    rr = fmaf(r, r, rr);
  }
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] = ~w[k];
  return rr;
}
template <int D, int BITS, typename T>
__global__ void __launch_bounds__(kRowThreads, 1) encode_rows_kernel(EncodeParams p) {
  constexpr int NJ = D / 32;
  constexpr int OPB = kTileVec * D * 2;           // bytes of one bf16 [128 x D] operand
  constexpr int SB = D * D * 2;                   // bytes of S [m x d] bf16
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t mbar[2];
  __shared__ uint32_t tmem_slot;
  uint8_t* base = raw + ((1024 - (tqtc::smem_u32(raw) & 1023)) & 1023);
  uint8_t* s_op = base;                           // S, K-major SW128 (rows = sketch index)

  const int tid = threadIdx.x, warp = tid >> 5;
  const int g = tid >> 7, t = tid & (kGroupThreads - 1);   // group, row in the tile
  uint8_t* r_hi = base + SB + g * 2 * OPB;       // this group's residual tile, hi bf16 piece
  uint8_t* r_lo = r_hi + OPB;                     // lo bf16 piece
  // bf16 inputs: each thread prefetches its row of the group's next tile
  // into shared memory (16-byte cp.async, chunk c stored at c ^ (t & 15) so
  // the row reads spread over the banks)
  constexpr bool kStage = sizeof(T) == 2;
  constexpr int RB = D * static_cast<int>(sizeof(T));   // bytes per row
  uint8_t* xstage = base + SB + 4 * OPB + g * kTileVec * RB + t * RB;
  auto prefetch_row = [&](int64_t tile) {
    if constexpr (kStage) {
      const int64_t r = tile * kTileVec + t;
      if (tile < (p.n + kTileVec - 1) / kTileVec && r < p.n) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(static_cast<const T*>(p.x) + r * p.ld);
#pragma unroll
        for (int c = 0; c < RB / 16; ++c) tqdev::cp_async16(xstage + 16 * (c ^ (t & (RB / 16 - 1))), src + 16 * c, 16);
      }
      tqdev::cp_async_commit();
    }
  };

  for (int c = tid; c < SB / 16; c += blockDim.x) tqdev::cp_async16(s_op + 16 * c, p.s_op + 8 * c, 16);
  tqdev::cp_async_commit();
  if (tid < 2) tqtc::mbar_init(&mbar[tid], 1);
  if (warp == 0) tqtc::tmem_alloc(&tmem_slot, 2 * D);
  tqdev::cp_async_wait<0>();
  tqtc::fence_before_sync();
  __syncthreads();
  tqtc::fence_after_sync();
  const uint32_t tmem = tmem_slot + g * D + (static_cast<uint32_t>(t & ~31) << 16);   // lane block of this warp
  const uint32_t idesc = tqtc::idesc_bf16_f32(kTileVec, D);
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  float tp[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) tp[k] = p.tpos[k];
  const int64_t n_tiles = (p.n + kTileVec - 1) / kTileVec;
  // swizzled row base of this thread's row in the residual operands
  const uint32_t rowbase = static_cast<uint32_t>((t >> 3) * 1024 + (t & 7) * 128);
  const uint32_t vx = t & 7;
  uint32_t phase = 0;

  prefetch_row(2 * static_cast<int64_t>(blockIdx.x) + g);
  for (int64_t tile = 2 * static_cast<int64_t>(blockIdx.x) + g; tile < n_tiles; tile += 2 * gridDim.x) {
    const int64_t row = tile * kTileVec + t;
    bool valid = row < p.n;
    float u[D];
    float nrm = 0.f, rr = 0.f;
    if constexpr (kStage) {
      // this thread's row (its own cp.async group), then the next tile's row
      tqdev::cp_async_wait<0>();
      if (valid) {
#pragma unroll
        for (int c = 0; c < RB / 16; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(xstage + 16 * (c ^ (t & (RB / 16 - 1))));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            u[8 * c + 2 * q] = __uint_as_float(w[q] << 16);
            u[8 * c + 2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
          }
        }
      }
      prefetch_row(tile + 2 * gridDim.x);
    }
    if (valid) {
      if constexpr (!kStage) load_row<D, T>(static_cast<const T*>(p.x) + row * p.ld, u);
      if (p.rope) {
        const int64_t pos = p.pos ? p.pos[row] : p.pos_offset + row % p.pos_period;
        if (pos < 0 || pos >= p.rope_max_pos) {
          valid = false;
          p.norms[row * p.out_stride] = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
        } else {
          // cos/sin(pos theta_i) from the two-level tables (angle addition)
          const float4* hi = reinterpret_cast<const float4*>(p.rope_hi + (pos >> kRopeLoBits) * (D / 2));
          const float4* lo = reinterpret_cast<const float4*>(p.rope_lo + (pos & (kRopeLoRows - 1)) * (D / 2));
#pragma unroll
          for (int c = 0; c < D / 4; ++c) {
            if ((c & 7) == 0) asm volatile("" ::: "memory");   // bound the loads in flight (registers)
            const float4 a = __ldg(hi + c), b = __ldg(lo + c);
            const float c0 = a.x * b.x - a.y * b.y, s0 = a.y * b.x + a.x * b.y;
            const float c1 = a.z * b.z - a.w * b.w, s1 = a.w * b.z + a.z * b.w;
            const int i0 = 2 * c, i1 = 2 * c + 1;
            const float x0 = u[i0], y0 = u[i0 + D / 2], x1 = u[i1], y1 = u[i1 + D / 2];
            u[i0] = x0 * c0 - y0 * s0;
            u[i0 + D / 2] = y0 * c0 + x0 * s0;
            u[i1] = x1 * c1 - y1 * s1;
            u[i1 + D / 2] = y1 * c1 + x1 * s1;
          }
        }
      }
    }
    if (valid) {
      float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < D; ++i) {
        ss[i & 3] = fmaf(u[i], u[i], ss[i & 3]);
        u[i] *= p.dsg[i];
      }
      nrm = sqrtf((ss[0] + ss[1]) + (ss[2] + ss[3]));
      fwht_regs<D>(u);
      const float scale = (nrm > 0.f ? 1.0f / nrm : 0.f) * inv_sqrt_d;
#pragma unroll
      for (int i = 0; i < D; ++i) u[i] = fmaf(u[i], scale, 0.f);   // unit-vector coordinates, -0 -> +0
      float nl[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) nl[k] = nrm * p.lpos[k];
      uint32_t words[BITS][NJ];
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        uint32_t w[BITS];
        rr += quantize32<BITS>(u + 32 * j, tp, nl, nrm, w);
#pragma unroll
        for (int k = 0; k < BITS; ++k) words[k][j] = w[k];
      }
      if (p.sign_res) {   // mean |r_i| in place of ||r||
        float ra = 0.f;
#pragma unroll
        for (int i = 0; i < D; ++i) ra += fabsf(u[i]);
        rr = ra * (1.f / D);
      } else {
        rr = sqrtf(rr);
      }
      uint32_t* crec = p.codes + row * p.out_stride * (BITS * NJ);   // 4-byte aligned records
#pragma unroll
      for (int k = 0; k < BITS; ++k)
#pragma unroll
        for (int j = 0; j < NJ; ++j) crec[k * NJ + j] = words[k][j];
      p.norms[row * p.out_stride] = make_float2(nrm, rr);
    } else {
#pragma unroll
      for (int i = 0; i < D; ++i) u[i] = 0.f;
    }
    // residual as bf16 hi + lo, row t of this group's A operand (16-byte chunks)
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      uint32_t h[4], l[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = u[8 * c + 2 * q], b = u[8 * c + 2 * q + 1];
        __nv_bfloat162 hb = __floats2bfloat162_rn(a, b);
        const uint32_t hbits = *reinterpret_cast<uint32_t*>(&hb);
        __nv_bfloat162 lb =
            __floats2bfloat162_rn(a - __uint_as_float(hbits << 16), b - __uint_as_float(hbits & 0xFFFF0000u));
        h[q] = hbits;
        l[q] = *reinterpret_cast<uint32_t*>(&lb);
      }
      const uint32_t off = (c >> 3) * (kTileVec * 128) + rowbase + ((((c & 7) ^ vx)) << 4);
      *reinterpret_cast<uint4*>(r_hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<uint4*>(r_lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
    // ---- S r of the tile on the tensor core (one thread of the group issues)
    tqtc::fence_smem_to_async();
    tqtc::fence_before_sync();
    group_sync(g);
    if (t == 0) {
      tqtc::fence_after_sync();
      const uint32_t dacc = tmem_slot + g * D;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tqtc::mma_bf16_ss(dacc, tqtc::sw128_desc_kstep(tqtc::smem_u32(r_hi), ks, kTileVec),
                          tqtc::sw128_desc_kstep(tqtc::smem_u32(s_op), ks, D), idesc, ks > 0);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tqtc::mma_bf16_ss(dacc, tqtc::sw128_desc_kstep(tqtc::smem_u32(r_lo), ks, kTileVec),
                          tqtc::sw128_desc_kstep(tqtc::smem_u32(s_op), ks, D), idesc, true);
      tqtc::mma_commit(&mbar[g]);
    }
    const bool ok = tqtc::mbar_wait(&mbar[g], phase, kWaitLimit);
    phase ^= 1;
    tqtc::fence_after_sync();
    // ---- sign bits of row t: lane t of the accumulator
    uint32_t sw[NJ];
#pragma unroll
    for (int c = 0; c < NJ; ++c) {
      float val[32];
      tqtc::tmem_ld32(tmem + 32 * c, val);
      uint32_t w = 0;
#pragma unroll
      for (int b = 31; b >= 0; --b) w = (w << 1) | (val[b] >= 0.f ? 1u : 0u);
      sw[c] = ok ? w : 0u;
    }
    if (row < p.n) {
      uint32_t* srec = p.signs + row * p.out_stride * NJ;
#pragma unroll
      for (int c = 0; c < NJ; ++c) srec[c] = sw[c];
      if (!ok) p.norms[row * p.out_stride] = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
    }
    tqtc::fence_before_sync();
    group_sync(g);
  }
  tqtc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tqtc::tmem_free(tmem_slot, 2 * D);
}

// Codes of the 32 coordinates held as y[m] = (c 2m, c 2m+1) (unit-vector
// coordinates, never -0): as quantize32, with the residual and its square
// sum formed two at a time (fp32x2).  Returns the sum of squared residuals.
template <int BITS>
__device__ __forceinline__ float quantize32_x2(float2* y, const float (&tp)[4], const float (&nl)[4], float norm,
                                               uint32_t (&w)[BITS]) {
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] = 0;
  const float2 norm2 = make_float2(norm, norm);
  // 2 bits: level = sign(v) (mid + sign(|v| - t_0) half), both signs taken
  // from sign bits the plane words already use (mid + half = nl[1] and
  // mid - half = nl[0] within an ulp)
  const uint32_t mid_b = __float_as_uint(0.5f * (nl[0] + nl[1])), half_b = __float_as_uint(0.5f * (nl[1] - nl[0]));
  float2 rr = make_float2(0.f, 0.f);
#pragma unroll
  for (int m = 15; m >= 0; --m) {
    float c[2];
#pragma unroll
    for (int e = 1; e >= 0; --e) {
      const float v = e ? y[m].y : y[m].x;
      const uint32_t sy = __float_as_uint(v);
      const float a = fabsf(v);
      if constexpr (BITS == 1) {
        w[0] = __funnelshift_l(sy, w[0], 1);
        c[e] = -copysignf(nl[0], v);
      } else if constexpr (BITS == 2) {
        const uint32_t s0 = __float_as_uint(a - tp[0]);
        const uint32_t x = sy ^ s0;
        w[1] = __funnelshift_l(sy, w[1], 1);
        w[0] = __funnelshift_l(x, w[0], 1);
        c[e] = -(__uint_as_float((sy & 0x80000000u) | mid_b) + __uint_as_float((x & 0x80000000u) | half_b));
      } else {
        const uint32_t s0 = __float_as_uint(a - tp[0]), s1 = __float_as_uint(a - tp[1]),
                       s2 = __float_as_uint(a - tp[2]);
        w[2] = __funnelshift_l(sy, w[2], 1);
        w[1] = __funnelshift_l(sy ^ s1, w[1], 1);
        w[0] = __funnelshift_l(sy ^ s0 ^ s1 ^ s2, w[0], 1);
        const float nmag = a >= tp[2] ? nl[3] : (a >= tp[1] ? nl[2] : (a >= tp[0] ? nl[1] : nl[0]));
        c[e] = -copysignf(nmag, v);
      }
    }
    const float2 r = __ffma2_rn(norm2, y[m], make_float2(c[0], c[1]));
    y[m] = r;
    rr = __ffma2_rn(r, r, rr);
  }
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] = ~w[k];
  return rr.x + rr.y;
}

// 2 pi = 6 + kC2 + kC3 (kC2 + kC3 within about 1e-17 of 2 pi - 6): with
// k < 2^22, k * 6 is exact and the three-term reduction of a RoPE angle
// (Cody and Waite's method) keeps its error near 2^-22.
constexpr double kTwoPiMinus6 = 0.28318530717958647692528676655900576839433879875021;
constexpr float kC2 = static_cast<float>(kTwoPiMinus6);
constexpr float kC3 = static_cast<float>(kTwoPiMinus6 - static_cast<double>(kC2));
constexpr float kInvTwoPi = 0.15915494309189533577f;
// Largest RoPE position the tensor-core encode takes: positions are exact as
// float and k = rint(angle / 2 pi) < 2^22 for every frequency (theta <= 1).
constexpr int64_t kPairsMaxRopePos = int64_t(1) << 22;

// ===========================================================================
// Rotation on the tensor core (d = 64 or 128, large batches).  y = H D x is
// a dense d x d contraction with exact +-1 entries, so each 128-row tile
// is rotated by tcgen05 MMAs against H D resident in shared memory, and the
// CUDA cores keep only RoPE, the codes, the residual and the sign bits.
//
// One CTA per SM runs two groups of 8 warps; each group owns a tile at a
// time (its own staging / operand buffers, tensor-memory columns, mbarriers
// and named barrier), so one group's tensor-core work and waits overlap the
// other's CUDA-core work.  S and H D are shared.  Per tile:
//  1. the input tile arrives by 2-D TMA (128-byte swizzle) into the group's
//     operand buffer, requested one tile ahead;
//  2. SPLIT (RoPE or fp32 input): thread pairs (row t, half h) load the row,
//     take ||x|| (before RoPE: a rotation keeps it), apply RoPE, scale by a
//     power of two near 1 / ||x|| and write fp16 hi + lo pieces (22 bits;
//     bf16 pieces, 2^-17, would move ||r|| by up to ~8e-6 ||x||) as the A
//     operand; otherwise (bf16 without RoPE) the staged tile is the A
//     operand as it stands (against bf16 H D, exact products);
//  3. y = A (H D)^T into tensor memory (fp32);
//  4. thread pairs (TMEM lane = row, column half) read y, form the unit
//     coordinates y / (||x|| sqrt d), the codes and the residual (fp32x2),
//     and write the residual as bf16 hi + lo over the A operand;
//  5. S r into the same tensor-memory columns; the sign bits are read back.
// SGN (sign-residual records, S = I): steps 4-5 keep no residual operand and
// no S r product; the sign bits of r come straight from the registers and the
// group's next tile is requested as soon as y has been read.
// ===========================================================================
constexpr int kTcThreads = 512;   // two groups of 8 warps

template <int D, int BITS, typename T, bool SPLIT, bool SGN>
__global__ void __launch_bounds__(kTcThreads, D == 64 ? 2 : 1) encode_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                 EncodeParams p) {
  static_assert(SPLIT || sizeof(T) == 2, "fp32 input needs the split path");
  static_assert(D == 64 || D == 128, "tensor-core encode: d = 64 or 128");
  constexpr int OPB = kTileVec * D * 2;           // one 16-bit [128 x d] operand (32 KB at d = 128)
  constexpr int SOPB = D * D * 2;                 // S or H D: one 16-bit [d x d] operand
  constexpr int HC = D / 4;                       // phase 2: coordinates per thread in each half of a row
  constexpr int NJ = D / 32;                      // 32-bit words per plane
  constexpr int kBoxCols = 128 / static_cast<int>(sizeof(T));
  constexpr int kBoxes = D / kBoxCols;
  constexpr uint32_t kXBytes = kTileVec * D * sizeof(T);
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t mb_x[2], mb_y[2], mb_s[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int s_fail[2];
  __shared__ __align__(16) float2 thh_s[D / 4];
  __shared__ __align__(16) float2 thl_s[D / 4];
  __shared__ float xnrm[2][2][kTileVec];          // per group: ||x|| (SPLIT) or partial sums of squares
  __shared__ float xrr[2][2][kTileVec];           // per group: partial sums of squared residuals
  uint8_t* base = raw + ((1024 - (tqtc::smem_u32(raw) & 1023)) & 1023);
  uint8_t* s_op = base;
  uint8_t* hd_op = base + SOPB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = warp >> 3, gw = warp & 7, gt = tid & 255;
  uint8_t* a_hi = base + 2 * SOPB + g * 2 * OPB;
  uint8_t* a_lo = a_hi + OPB;
  uint8_t* xs = a_hi;   // staged input tile (bf16: a_hi; fp32: a_hi and a_lo)
  const int64_t n_tiles = (p.n + kTileVec - 1) / kTileVec;
  const int64_t tstep = 2 * static_cast<int64_t>(gridDim.x);
  auto gsync = [&]() { asm volatile("bar.sync %0, 256;\n" ::"r"(1 + g) : "memory"); };
  auto issue_x = [&](int64_t tl) {
    tqtc::mbar_arrive_expect_tx(&mb_x[g], kXBytes);
#pragma unroll
    for (int b = 0; b < kBoxes; ++b)
      tqtc::tma_load_2d(xs + b * (kTileVec * 128), &xmap, b * kBoxCols, static_cast<int>(tl * kTileVec), &mb_x[g]);
  };
  for (int c = tid; c < 2 * SOPB / 16; c += blockDim.x)
    tqdev::cp_async16(base + 16 * c, c < SOPB / 16 ? p.s_op + 8 * c : p.hd_op + 8 * (c - SOPB / 16), 16);
  tqdev::cp_async_commit();
  if (tid < D / 4) {
    thh_s[tid] = make_float2(p.theta[2 * tid].x, p.theta[2 * tid + 1].x);
    thl_s[tid] = make_float2(p.theta[2 * tid].y, p.theta[2 * tid + 1].y);
  }
  if (tid == 0) {
    s_fail[0] = s_fail[1] = 0;
    for (int i = 0; i < 2; ++i) {
      tqtc::mbar_init(&mb_x[i], 1);
      tqtc::mbar_init(&mb_y[i], 1);
      tqtc::mbar_init(&mb_s[i], 1);
    }
  }
  if (warp == 0) tqtc::tmem_alloc(&tmem_slot, 2 * D);
  tqdev::cp_async_wait<0>();
  tqtc::fence_smem_to_async();
  tqtc::fence_before_sync();
  __syncthreads();
  tqtc::fence_after_sync();
  int64_t tile = 2 * static_cast<int64_t>(blockIdx.x) + g;
  if (gt == 0 && tile < n_tiles) issue_x(tile);
  const uint32_t tm = tmem_slot + D * g;                    // y, then S r: d columns per group
  const uint32_t tm_lane = static_cast<uint32_t>(32 * (gw & 3)) << 16;
  constexpr uint32_t idy = SPLIT ? tqtc::idesc_f16_f32(kTileVec, D) : tqtc::idesc_bf16_f32(kTileVec, D);
  constexpr uint32_t ids = tqtc::idesc_bf16_f32(kTileVec, D);
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  const float2 m1 = make_float2(-1.f, -1.f);
  float tp[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) tp[k] = p.tpos[k];
  // phase-2 mapping (SPLIT): row t2 of the tile, coordinates {HC h2 + i, d/2 + HC h2 + i}, i < HC
  const int t2 = 32 * (gw & 3) + 16 * (gw >> 2) + (lane & 15), h2 = lane >> 4;
  const uint32_t rowbase2 = static_cast<uint32_t>((t2 >> 3) * 1024 + (t2 & 7) * 128);
  // phase-4 mapping: row r4 = tensor-memory lane, coordinates d/2 c4 .. d/2 c4 + d/2 - 1
  const int r4 = 32 * (gw & 3) + lane, c4 = gw >> 2;
  const uint32_t rowbase4 = static_cast<uint32_t>((r4 >> 3) * 1024 + (r4 & 7) * 128);
  uint32_t ph_x = 0, ph_y = 0, ph_s = 0;
  const float qnan = __int_as_float(0x7fc00000);

  for (; tile < n_tiles; tile += tstep) {
    const bool failed = s_fail[g] != 0;   // written before the previous iteration's last barrier
    const bool ok_x = !failed && tqtc::mbar_wait(&mb_x[g], ph_x, kWaitLimit);
    ph_x ^= 1;
    if constexpr (SPLIT) {
      // ---- 2. row t2 into registers, ||x||, RoPE, fp16 hi + lo A operand
      const int64_t row = tile * kTileVec + t2;
      bool valid = row < p.n && ok_x;
      // v[HC/2 s + m] = coordinates (d/2 s + HC h2 + 2m, + 1); a staged row is
      // 128-byte boxes of 16-byte chunks, chunk c of a box at c ^ (row % 8)
      constexpr int NV = HC;   // float2 per thread
      float2 v[NV];
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int sh = 0; sh < 2; ++sh)
#pragma unroll
          for (int q = 0; q < HC / 8; ++q) {
            // chunk of 8 coordinates: box, chunk within the box
            const int box = D == 128 ? sh : 0, cb = D == 128 ? 4 * h2 + q : 4 * sh + 2 * h2 + q;
            const uint4 w4 = *reinterpret_cast<const uint4*>(xs + box * (kTileVec * 128) + t2 * 128 +
                                                             ((cb ^ (t2 & 7)) << 4));
            const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              v[(HC / 2) * sh + 4 * q + e] =
                  make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
          }
      } else {
#pragma unroll
        for (int sh = 0; sh < 2; ++sh)
#pragma unroll
          for (int q = 0; q < HC / 4; ++q) {
            // chunk of 4 coordinates: box, chunk within the box
            const int box = D == 128 ? 2 * sh + h2 : sh, cb = D == 128 ? q : 4 * h2 + q;
            const float4 f = *reinterpret_cast<const float4*>(xs + box * (kTileVec * 128) + t2 * 128 +
                                                              ((cb ^ (t2 & 7)) << 4));
            v[(HC / 2) * sh + 2 * q] = make_float2(f.x, f.y);
            v[(HC / 2) * sh + 2 * q + 1] = make_float2(f.z, f.w);
          }
      }
      float ss;
      {
        float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int m = 0; m < NV; ++m) a2 = __ffma2_rn(v[m], v[m], a2);
        ss = a2.x + a2.y;
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 16);
      if (valid && p.rope) {
        const int64_t pos = p.pos ? p.pos[row] : p.pos_offset + row % p.pos_period;
        if (pos < 0 || pos >= p.rope_max_pos) {
          valid = false;
        } else {
          // pairs (v[m], v[HC/2 + m]) turn by pos * theta_j, j = HC h2 + 2m (+1):
          // angle pos theta_hi + pos theta_lo, reduced by 2 pi in three terms
          // (k negated: rint is odd), then sin / cos on [-pi, pi]
          const float pf = static_cast<float>(pos);   // exact: pos < 2^22
          const float2 pf2 = make_float2(pf, pf), npf2 = make_float2(-pf, -pf);
          const float2 q2c = make_float2(-kInvTwoPi, -kInvTwoPi), six2 = make_float2(6.f, 6.f);
          const float2 c2c = make_float2(kC2, kC2), c3c = make_float2(kC3, kC3);
#pragma unroll
          for (int m = 0; m < HC / 2; ++m) {
            if ((m & 3) == 0) asm volatile("" ::: "memory");   // bound the loads in flight (registers)
            const float2 thh = thh_s[(HC / 2) * h2 + m], thl = thl_s[(HC / 2) * h2 + m];
            const float2 ah = __fmul2_rn(pf2, thh);
            const float2 e = __ffma2_rn(npf2, thh, ah);
            const float2 nal = __ffma2_rn(npf2, thl, e);
            const float2 q = __fmul2_rn(ah, q2c);
            const float2 kn = make_float2(rintf(q.x), rintf(q.y));
            float2 r = __ffma2_rn(kn, six2, ah);
            r = __ffma2_rn(kn, c2c, r);
            r = __ffma2_rn(kn, c3c, r);
            r = __ffma2_rn(nal, m1, r);
            float s0, c0, s1, c1;
            __sincosf(r.x, &s0, &c0);
            __sincosf(r.y, &s1, &c1);
            const float2 sn = make_float2(s0, s1), cs = make_float2(c0, c1);
            const float2 x = v[m], y = v[HC / 2 + m];
            v[m] = __ffma2_rn(y, __fmul2_rn(sn, m1), __fmul2_rn(x, cs));
            v[HC / 2 + m] = __ffma2_rn(x, sn, __fmul2_rn(y, cs));
          }
        }
      }
      const float nrm = sqrtf(ss);
      // a power of two near 1 / ||x|| keeps the fp16 pieces in range (exact scaling)
      float sc = 0.f;
      if (valid && nrm > 0.f) {
        int e;
        frexpf(nrm, &e);
        sc = ldexpf(1.f, -e);
      }
      if (h2 == 0) xnrm[g][0][t2] = valid ? nrm : qnan;
      if (!valid && row < p.n && h2 == 0) p.norms[row * p.out_stride] = make_float2(qnan, qnan);
      const float2 sc2 = make_float2(sc, sc);
      gsync();   // every row is in registers: the staging buffer takes the A operand
#pragma unroll
      for (int sh = 0; sh < 2; ++sh)
#pragma unroll
        for (int q = 0; q < HC / 8; ++q) {
          uint32_t hv[4], lv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = __fmul2_rn(v[(HC / 2) * sh + 4 * q + e], sc2);
            const __half2 hh = __floats2half2_rn(x.x, x.y);
            const float2 lo = __ffma2_rn(__half22float2(hh), m1, x);
            const __half2 lh = __floats2half2_rn(lo.x, lo.y);
            hv[e] = *reinterpret_cast<const uint32_t*>(&hh);
            lv[e] = *reinterpret_cast<const uint32_t*>(&lh);
          }
          // 16-byte chunk of the K-major operand row: K block, chunk within it
          const int kb = D == 128 ? sh : 0, cb = D == 128 ? 4 * h2 + q : 4 * sh + 2 * h2 + q;
          const uint32_t off = kb * (kTileVec * 128) + rowbase2 + ((cb ^ (t2 & 7)) << 4);
          *reinterpret_cast<uint4*>(a_hi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
          *reinterpret_cast<uint4*>(a_lo + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
        }
      tqtc::fence_smem_to_async();
    }
    const int64_t row = tile * kTileVec + r4;
    if constexpr (!SPLIT) {
      // ||x||^2 of row r4, this thread's d/2 coordinates of the staged bf16 tile
      float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        const int box = D == 128 ? c4 : 0, cb = D == 128 ? j : 4 * c4 + j;
        const uint4 w4 = *reinterpret_cast<const uint4*>(xs + box * (kTileVec * 128) + rowbase4 +
                                                         ((cb ^ (r4 & 7)) << 4));
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
          a2 = __ffma2_rn(x, x, a2);
        }
      }
      xnrm[g][c4][r4] = a2.x + a2.y;
    }
    // ---- 3. y = A (H D)^T
    tqtc::fence_before_sync();
    gsync();
    if (gt == 0 && !failed) {
      tqtc::fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tqtc::mma_bf16_ss(tm, tqtc::sw128_desc_kstep(tqtc::smem_u32(a_hi), ks, kTileVec),
                          tqtc::sw128_desc_kstep(tqtc::smem_u32(hd_op), ks, D), idy, ks > 0);
      if constexpr (SPLIT) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tqtc::mma_bf16_ss(tm, tqtc::sw128_desc_kstep(tqtc::smem_u32(a_lo), ks, kTileVec),
                            tqtc::sw128_desc_kstep(tqtc::smem_u32(hd_op), ks, D), idy, true);
      }
      tqtc::mma_commit(&mb_y[g]);
    }
    // ---- 4. codes and residual of row r4, coordinates 64 c4 ..
    float nrm, scale;
    bool valid;
    if constexpr (SPLIT) {
      nrm = xnrm[g][0][r4];
      valid = row < p.n && !isnan(nrm);
      float sc = 0.f;
      if (valid && nrm > 0.f) {
        int e;
        frexpf(nrm, &e);
        sc = ldexpf(1.f, -e);
      }
      // y holds H D (sc x): the unit coordinates are y / (sc ||x|| sqrt d)
      scale = valid && nrm > 0.f ? 1.f / (sc * nrm) * inv_sqrt_d : 0.f;
    } else {
      nrm = sqrtf(xnrm[g][0][r4] + xnrm[g][1][r4]);
      valid = row < p.n && ok_x;
      scale = valid && nrm > 0.f ? 1.f / nrm * inv_sqrt_d : 0.f;
      if (!valid && row < p.n && c4 == 0) p.norms[row * p.out_stride] = make_float2(qnan, qnan);
    }
    const bool ok_y = !failed && tqtc::mbar_wait(&mb_y[g], ph_y, kWaitLimit);
    ph_y ^= 1;
    tqtc::fence_after_sync();
    constexpr int NU = D / 4;   // float2 per thread
    float2 u[NU];   // u[m] = coordinates (d/2 c4 + 2m, + 1)
    if constexpr (D == 128 && SPLIT) {   // both 32-column loads under one wait (the key launches)
      float y0[32], y1[32];
      tqtc::tmem_ld32x2(tm + tm_lane + 64 * c4, tm + tm_lane + 64 * c4 + 32, y0, y1);
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        u[m] = make_float2(y0[2 * m], y0[2 * m + 1]);
        u[16 + m] = make_float2(y1[2 * m], y1[2 * m + 1]);
      }
    } else {
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        float y[32];
        tqtc::tmem_ld32(tm + tm_lane + (D / 2) * c4 + 32 * h, y);
#pragma unroll
        for (int m = 0; m < 16; ++m) u[16 * h + m] = make_float2(y[2 * m], y[2 * m + 1]);
      }
    }
    {
      const float2 sc2 = make_float2(scale, scale), z2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int m = 0; m < NU; ++m) u[m] = __ffma2_rn(u[m], sc2, z2);   // unit-vector coordinates, -0 -> +0
    }
    const float nv = valid ? nrm : 0.f;
    float nl[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) nl[k] = nv * p.lpos[k];
    uint32_t wq[D / 64][BITS];   // words (d/64) c4 + h of each plane
    float rr = 0.f;
#pragma unroll
    for (int h = 0; h < D / 64; ++h) rr += quantize32_x2<BITS>(u + 16 * h, tp, nl, nv, wq[h]);
    if (p.sign_res) {   // sum of |r_i| over this thread's d/2 coordinates in place of sum r_i^2
      float2 ra = make_float2(0.f, 0.f);
#pragma unroll
      for (int m = 0; m < NU; ++m) ra = __fadd2_rn(ra, make_float2(fabsf(u[m].x), fabsf(u[m].y)));
      rr = ra.x + ra.y;
    }
    xrr[g][c4][r4] = rr;
    if (valid && ok_y) {
      uint32_t* crec = p.codes + row * p.out_stride * (BITS * NJ);   // 4-byte aligned records
#pragma unroll
      for (int k = 0; k < BITS; ++k)
#pragma unroll
        for (int h = 0; h < D / 64; ++h) crec[k * NJ + (D / 64) * c4 + h] = wq[h][k];
    }
    if constexpr (SGN) {
      // sign-residual records: S is the identity, so the sign bits are those
      // of r itself, taken from the registers (no S r product, no residual
      // operand); the staged tile and y are consumed, so the group's next
      // tile is requested at once
      uint32_t ws[D / 64];
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t w = 0;
#pragma unroll
        for (int b = 31; b >= 0; --b) {
          const float2 r = u[16 * c + (b >> 1)];
          w = __funnelshift_l(__float_as_uint((b & 1) ? r.y : r.x), w, 1);
        }
        ws[c] = ~w;
      }
      tqtc::fence_before_sync();
      gsync();   // the partner half's sum of |r_i| (xrr) is visible
      if (valid && ok_y && c4 == 0) p.norms[row * p.out_stride] = make_float2(nrm, (rr + xrr[g][1][r4]) * (1.f / D));
      if (!ok_y || !ok_x) s_fail[g] = 1;
      if (gt == 0 && ok_y && tile + tstep < n_tiles) issue_x(tile + tstep);
      if (row < p.n) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) p.signs[row * p.out_stride * NJ + (D / 64) * c4 + c] = ok_y ? ws[c] : 0u;
        if (!ok_y && c4 == 0) p.norms[row * p.out_stride] = make_float2(qnan, qnan);
      }
    } else {
      // residual (zero on absent rows) as bf16 hi + lo over the A operand, row r4
      // (the staged tile was read before the barrier ahead of the products)
  #pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        uint32_t hv[4], lv[4];
  #pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 r = u[4 * j + e];
          __nv_bfloat162 hb2 = __floats2bfloat162_rn(r.x, r.y);
          const uint32_t hbits = *reinterpret_cast<uint32_t*>(&hb2);
          const float2 lo =
              __ffma2_rn(make_float2(__uint_as_float(hbits << 16), __uint_as_float(hbits & 0xFFFF0000u)), m1, r);
          __nv_bfloat162 lb = __floats2bfloat162_rn(lo.x, lo.y);
          hv[e] = hbits;
          lv[e] = *reinterpret_cast<uint32_t*>(&lb);
        }
        const int kb = D == 128 ? c4 : 0, cb = D == 128 ? j : 4 * c4 + j;
        const uint32_t off = kb * (kTileVec * 128) + rowbase4 + ((cb ^ (r4 & 7)) << 4);
        *reinterpret_cast<uint4*>(a_hi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<uint4*>(a_lo + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
      }
      // ---- 5. S r of the tile, into the columns y has left
      tqtc::fence_smem_to_async();
      tqtc::fence_before_sync();
      gsync();
      if (gt == 0 && !failed) {
        tqtc::fence_after_sync();
  #pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tqtc::mma_bf16_ss(tm, tqtc::sw128_desc_kstep(tqtc::smem_u32(a_hi), ks, kTileVec),
                            tqtc::sw128_desc_kstep(tqtc::smem_u32(s_op), ks, D), ids, ks > 0);
  #pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tqtc::mma_bf16_ss(tm, tqtc::sw128_desc_kstep(tqtc::smem_u32(a_lo), ks, kTileVec),
                            tqtc::sw128_desc_kstep(tqtc::smem_u32(s_op), ks, D), ids, true);
        tqtc::mma_commit(&mb_s[g]);
      }
      if (valid && ok_y && c4 == 0)
        p.norms[row * p.out_stride] =
            make_float2(nrm, p.sign_res ? (rr + xrr[g][1][r4]) * (1.f / D) : sqrtf(rr + xrr[g][1][r4]));
      const bool ok = ok_y && tqtc::mbar_wait(&mb_s[g], ph_s, kWaitLimit);
      ph_s ^= 1;
      tqtc::fence_after_sync();
      if (!ok || !ok_x) s_fail[g] = 1;
      // the products have read the operand buffer: it takes the group's next tile
      if (gt == 0 && ok && tile + tstep < n_tiles) issue_x(tile + tstep);
      // sign bits of S r: complemented fp32 sign bits, one funnel shift each
      // (an exact -0 projection reads as negative, within the sign tolerance)
      {
        if constexpr (D == 128 && SPLIT) {   // both loads under one wait (the key launches)
          float val[2][32];
          tqtc::tmem_ld32x2(tm + tm_lane + 64 * c4, tm + tm_lane + 64 * c4 + 32, val[0], val[1]);
  #pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t w = 0;
  #pragma unroll
            for (int b = 31; b >= 0; --b) w = __funnelshift_l(__float_as_uint(val[c][b]), w, 1);
            if (row < p.n) p.signs[row * p.out_stride * NJ + 2 * c4 + c] = ok ? ~w : 0u;
          }
        } else {
  #pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            float val[32];
            tqtc::tmem_ld32(tm + tm_lane + (D / 2) * c4 + 32 * c, val);
            uint32_t w = 0;
  #pragma unroll
            for (int b = 31; b >= 0; --b) w = __funnelshift_l(__float_as_uint(val[b]), w, 1);
            if (row < p.n) p.signs[row * p.out_stride * NJ + (D / 64) * c4 + c] = ok ? ~w : 0u;
          }
        }
        if (!ok && c4 == 0 && row < p.n) p.norms[row * p.out_stride] = make_float2(qnan, qnan);
      }
    }
    tqtc::fence_before_sync();
    gsync();
  }
  tqtc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tqtc::tmem_free(tmem_slot, 2 * D);
}

template <int D, int BITS, typename T>
int launch_encode_rows(const EncodeParams& p, cudaStream_t stream) {
  // S + two groups x (hi, lo) residual tiles + (bf16) two staged input tiles:
  // 225 KB at d = 128
  const size_t stage = sizeof(T) == 2 ? 2 * static_cast<size_t>(kTileVec) * D * sizeof(T) : 0;
  const size_t smem = static_cast<size_t>(D) * D * 2 + 4 * static_cast<size_t>(kTileVec) * D * 2 + stage + 1024;
  auto kern = encode_rows_kernel<D, BITS, T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return TQ_ECUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (p.n + kTileVec - 1) / kTileVec;
  const int64_t pairs = (tiles + 1) / 2;
  const int blocks = static_cast<int>(pairs < sms ? pairs : sms);
  kern<<<blocks, kRowThreads, smem, stream>>>(p);
  return tq::launch_status();
}

// Batches below this many vectors take the low-latency warp-per-vector kernel.
constexpr int64_t kRowsKernelMinN = 16384;

template <int D, int BITS, typename T, bool SPLIT, bool SGN>
int launch_encode_tc_mode(const EncodeParams& p, const CUtensorMap& xmap, cudaStream_t stream) {
  // S, H D, 2 groups x (hi, lo): 193 KB at d = 128, 81 KB at d = 64
  const size_t smem = 2 * static_cast<size_t>(D) * D * 2 + 4 * static_cast<size_t>(kTileVec) * D * 2 + 1024;
  auto kern = encode_tc_kernel<D, BITS, T, SPLIT, SGN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return TQ_ECUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (p.n + kTileVec - 1) / kTileVec;
  const int64_t pairs = (tiles + 1) / 2;
  const int64_t slots = static_cast<int64_t>(sms) * (D == 64 ? 2 : 1);   // CTAs resident per SM
  const int blocks = static_cast<int>(pairs < slots ? pairs : slots);
  kern<<<blocks, kTcThreads, smem, stream>>>(xmap, p);
  return tq::launch_status();
}

template <int D, int BITS, typename T, bool SPLIT>
int launch_encode_tc(const EncodeParams& p, const CUtensorMap& xmap, cudaStream_t stream) {
  if (p.sign_res) return launch_encode_tc_mode<D, BITS, T, SPLIT, true>(p, xmap, stream);
  return launch_encode_tc_mode<D, BITS, T, SPLIT, false>(p, xmap, stream);
}

template <int D, int BITS, typename T>
int launch_encode_tcd(const EncodeParams& p, cudaStream_t stream) {
  // Positions past 2^22 (the in-kernel angle reduction's range) or more rows
  // than a TMA coordinate holds go to the table-driven one-thread kernel.
  if ((p.rope && p.rope_max_pos > kPairsMaxRopePos) || p.n >= (int64_t(1) << 31) || !p.hd_op)
    return launch_encode_rows<D, BITS, T>(p, stream);
  CUtensorMap xmap;
  if (!tq::make_tmap_2d(&xmap, p.x, static_cast<int>(sizeof(T)), p.n, D, p.ld, 128 / static_cast<int>(sizeof(T)),
                        kTileVec))
    return launch_encode_rows<D, BITS, T>(p, stream);
  if constexpr (sizeof(T) == 2) {
    if (!p.rope) return launch_encode_tc<D, BITS, T, false>(p, xmap, stream);
  }
  return launch_encode_tc<D, BITS, T, true>(p, xmap, stream);
}

template <int D, int BITS, typename T>
int launch_encode(const EncodeParams& p, cudaStream_t stream) {
  if (p.n <= kVecKernelMaxN) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.n));
    cfg.blockDim = dim3(D);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, encode_vec_kernel<D, BITS, T>, p) == cudaSuccess ? TQ_OK : TQ_ECUDA;
  }
  if (p.n < kRowsKernelMinN || p.out_rows) return launch_encode_warp<D, BITS, T>(p, stream);
  return launch_encode_tcd<D, BITS, T>(p, stream);
}

template <int D, int BITS, typename T>
int launch_encode_vec_pair(const EncodeParams& pk, const EncodeParams& pv, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pk.n), 2);
  cfg.blockDim = dim3(D);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, encode_vec_pair_kernel<D, BITS, T>, pk, pv) == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

template <int D, typename T>
int dispatch_vec_pair(int bits, const EncodeParams& pk, const EncodeParams& pv, cudaStream_t s) {
  switch (bits) {
    case 1: return launch_encode_vec_pair<D, 1, T>(pk, pv, s);
    case 2: return launch_encode_vec_pair<D, 2, T>(pk, pv, s);
    case 3: return launch_encode_vec_pair<D, 3, T>(pk, pv, s);
  }
  return TQ_EUNSUPPORTED;
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

namespace {

// Checks of one tq_quantize_kv call and its kernel parameters.
int make_encode_params(const tq_rotation* h, const void* x, int dtype, int64_t n, int64_t ld, const int64_t* pos,
                       int64_t pos_period, int64_t pos_offset, int apply_rope, uint8_t* codes, uint8_t* signs,
                       float* norms, int64_t out_stride, EncodeParams* out, const int64_t* out_rows = nullptr,
                       int64_t n_records = 0) {
  if (!h) return TQ_EINVAL;
  if (n < 0 || (dtype != TQ_F32 && dtype != TQ_BF16)) return TQ_EINVAL;
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
  p.out_rows = out_rows;
  p.n_records = n_records;
  fill_handle_fields(p, h);
  // H D for the tensor-core encode: fp16 when the rows are split (RoPE or fp32 input), else bf16
  p.hd_op = (apply_rope || dtype == TQ_F32) ? h->d_hd_f16 : h->d_hd_bf16;
  *out = p;
  return TQ_OK;
}

}  // namespace

extern "C" int tq_quantize_kv(const tq_rotation* h, const void* x, int dtype, int64_t n, int64_t ld,
                              const int64_t* pos, int64_t pos_period, int64_t pos_offset,
                              int apply_rope, uint8_t* codes, uint8_t* signs, float* norms,
                              int64_t out_stride, void* stream) {
  if (!h) return TQ_EINVAL;
  if (n < 0 || (dtype != TQ_F32 && dtype != TQ_BF16)) return TQ_EINVAL;
  if (n == 0) return TQ_OK;
  EncodeParams p{};
  const int st = make_encode_params(h, x, dtype, n, ld, pos, pos_period, pos_offset, apply_rope, codes, signs, norms,
                                    out_stride, &p);
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (h->d == 128)
    return dtype == TQ_F32 ? dispatch_bits<128, float>(h->bits, p, s) : dispatch_bits<128, __nv_bfloat16>(h->bits, p, s);
  if (h->d == 64)
    return dtype == TQ_F32 ? dispatch_bits<64, float>(h->bits, p, s) : dispatch_bits<64, __nv_bfloat16>(h->bits, p, s);
  return TQ_EUNSUPPORTED;
}

extern "C" int tq_quantize_kv_pair(const tq_rotation* hk, const void* xk, const tq_rotation* hv, const void* xv,
                                   int dtype, int64_t n, int64_t ld, const int64_t* pos, int64_t pos_period,
                                   int64_t pos_offset, int apply_rope, uint8_t* k_codes, uint8_t* k_signs,
                                   float* k_norms, uint8_t* v_codes, uint8_t* v_signs, float* v_norms,
                                   int64_t out_stride, void* stream) {
  if (!hk || !hv) return TQ_EINVAL;
  if (n < 0 || (dtype != TQ_F32 && dtype != TQ_BF16)) return TQ_EINVAL;
  if (n == 0) return TQ_OK;
  EncodeParams pk{}, pv{};
  int st = make_encode_params(hk, xk, dtype, n, ld, pos, pos_period, pos_offset, apply_rope, k_codes, k_signs,
                              k_norms, out_stride, &pk);
  if (st != TQ_OK) return st;
  if ((st = make_encode_params(hv, xv, dtype, n, ld, nullptr, 1, 0, 0, v_codes, v_signs, v_norms, out_stride, &pv)) !=
      TQ_OK)
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n <= kVecKernelMaxN && hk->d == hv->d && hk->bits == hv->bits && (hk->d == 128 || hk->d == 64)) {
    if (hk->d == 128)
      return dtype == TQ_F32 ? dispatch_vec_pair<128, float>(hk->bits, pk, pv, s)
                             : dispatch_vec_pair<128, __nv_bfloat16>(hk->bits, pk, pv, s);
    return dtype == TQ_F32 ? dispatch_vec_pair<64, float>(hk->bits, pk, pv, s)
                           : dispatch_vec_pair<64, __nv_bfloat16>(hk->bits, pk, pv, s);
  }
  st = tq_quantize_kv(hk, xk, dtype, n, ld, pos, pos_period, pos_offset, apply_rope, k_codes, k_signs, k_norms,
                      out_stride, stream);
  if (st != TQ_OK) return st;
  return tq_quantize_kv(hv, xv, dtype, n, ld, nullptr, 1, 0, 0, v_codes, v_signs, v_norms, out_stride, stream);
}

extern "C" int tq_quantize_kv_scatter(const tq_rotation* h, const void* x, int dtype, int64_t n, int64_t ld,
                                      const int64_t* pos, int64_t pos_period, int64_t pos_offset, int apply_rope,
                                      uint8_t* codes, uint8_t* signs, float* norms, const int64_t* out_rows,
                                      int64_t n_records, void* stream) {
  if (!h) return TQ_EINVAL;
  if (n < 0 || (dtype != TQ_F32 && dtype != TQ_BF16) || !out_rows || n_records < 1) return TQ_EINVAL;
  if (n == 0) return TQ_OK;
  EncodeParams p{};
  const int st = make_encode_params(h, x, dtype, n, ld, pos, pos_period, pos_offset, apply_rope, codes, signs, norms,
                                    1, &p, out_rows, n_records);
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (h->d == 128)
    return dtype == TQ_F32 ? dispatch_bits<128, float>(h->bits, p, s) : dispatch_bits<128, __nv_bfloat16>(h->bits, p, s);
  if (h->d == 64)
    return dtype == TQ_F32 ? dispatch_bits<64, float>(h->bits, p, s) : dispatch_bits<64, __nv_bfloat16>(h->bits, p, s);
  return TQ_EUNSUPPORTED;
}

extern "C" int tq_quantize_kv_pair_scatter(const tq_rotation* hk, const void* xk, const tq_rotation* hv,
                                           const void* xv, int dtype, int64_t n, int64_t ld, const int64_t* pos,
                                           int64_t pos_period, int64_t pos_offset, int apply_rope, uint8_t* k_codes,
                                           uint8_t* k_signs, float* k_norms, uint8_t* v_codes, uint8_t* v_signs,
                                           float* v_norms, const int64_t* out_rows, int64_t n_records,
                                           void* stream) {
  if (!hk || !hv) return TQ_EINVAL;
  if (n < 0 || (dtype != TQ_F32 && dtype != TQ_BF16) || !out_rows || n_records < 1) return TQ_EINVAL;
  if (n == 0) return TQ_OK;
  EncodeParams pk{}, pv{};
  int st = make_encode_params(hk, xk, dtype, n, ld, pos, pos_period, pos_offset, apply_rope, k_codes, k_signs,
                              k_norms, 1, &pk, out_rows, n_records);
  if (st != TQ_OK) return st;
  if ((st = make_encode_params(hv, xv, dtype, n, ld, nullptr, 1, 0, 0, v_codes, v_signs, v_norms, 1, &pv, out_rows,
                               n_records)) != TQ_OK)
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n <= kVecKernelMaxN && hk->d == hv->d && hk->bits == hv->bits && (hk->d == 128 || hk->d == 64)) {
    if (hk->d == 128)
      return dtype == TQ_F32 ? dispatch_vec_pair<128, float>(hk->bits, pk, pv, s)
                             : dispatch_vec_pair<128, __nv_bfloat16>(hk->bits, pk, pv, s);
    return dtype == TQ_F32 ? dispatch_vec_pair<64, float>(hk->bits, pk, pv, s)
                           : dispatch_vec_pair<64, __nv_bfloat16>(hk->bits, pk, pv, s);
  }
  st = tq_quantize_kv_scatter(hk, xk, dtype, n, ld, pos, pos_period, pos_offset, apply_rope, k_codes, k_signs, k_norms,
                              out_rows, n_records, stream);
  if (st != TQ_OK) return st;
  return tq_quantize_kv_scatter(hv, xv, dtype, n, ld, nullptr, 1, 0, 0, v_codes, v_signs, v_norms, out_rows,
                                n_records, stream);
}
