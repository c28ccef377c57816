// Dense fp32 contraction on the 5th-generation tensor core (tcgen05) by
// bf16 splitting: C[M][N] = A[M][K] B[N][K]^T with every fp32 operand given
// as bf16 pieces a = a_hi + a_lo (|a - a_hi - a_lo| <= 2^-17 |a|), and
//   C ~ A_hi B_hi^T + A_hi B_lo^T + A_lo B_hi^T      (fp32 accumulation)
// (the dropped A_lo B_lo^T term is below 2^-16 of each product).  With B
// exactly representable in bf16 (the QJL matrix) the B_lo term is absent.
//
// This serves the dense pieces of the codec - the rotation y = Pi x for a
// dense Pi ([TurboQuant] "Principe", Étape 1) and the sketch S r ([TurboQuant]
// "QJL") - where d is not a power of two and no fast transform exists.
//
// Kernel: persistent, one CTA per SM over 128 x 128 output tiles.  Operand
// tiles of 64 K-elements are loaded by TMA (2-D tensor maps, 128-byte
// swizzle, zero fill past the matrix edges) into a 3- or 4-stage ring (192
// KB); one thread issues the loads, one the MMAs (M = 128, N = 128, K = 16
// each), completion of a stage's MMAs frees it through tcgen05.commit on an
// mbarrier, and four epilogue warps drain each tile.  K tiles go round-robin
// to four fp32 accumulators in tensor memory (all 512 columns), summed in
// fp32 by the CUDA cores at the end: the tensor core's accumulation rounds
// toward zero, and with d = 1536 a single accumulator shrank the rotated
// coordinates by ~5e-6 relative; a quarter of the accumulation steps per
// accumulator keeps that bias near 1e-6.  Every wait is bounded; a tile whose
// wait runs out is written as NaN.  Each CTA loads its own tiles.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "tcgen05.cuh"
#include "tq_internal.h"

namespace {

constexpr int kGM = 128, kGN = 128, kGK = 64;
constexpr int kGAcc = 4;                     // tensor-memory accumulators (kGAcc * kGN = 512 columns)
constexpr int kGWaitLimit = 1 << 17;   // polls of about 9 us each: a wait gives up after about a second
constexpr int kATileBytes = kGM * kGK * 2;   // 16 KB
constexpr int kBTileBytes = kGN * kGK * 2;   // 16 KB

// Persistent form of the split-bf16 GEMM: one CTA per SM walks the output
// tiles (stride gridDim.x).  Warp 0 (one thread) streams every tile's K tiles
// through the TMA ring; warp 1 (one thread) issues the MMAs, and before each
// new tile waits until the epilogue has taken the previous tile's four
// accumulators out of tensor memory; warps 2-5 (tensor-memory lane quadrants
// warp % 4) wait for a tile's last MMA, sum its accumulators into registers,
// release tensor memory (128 arrivals on an mbarrier) and only then store,
// so the stores and the next tile's loads overlap the next tile's MMAs.
// Every wait is bounded; once one runs out, later tiles are written as NaN
// without waiting.
constexpr int kPThreads = 6 * 32;

template <bool BLO>
__global__ void __launch_bounds__(kPThreads, 1) tc_gemm_persistent_kernel(const __grid_constant__ CUtensorMap mAh,
                                                                         const __grid_constant__ CUtensorMap mAl,
                                                                         const __grid_constant__ CUtensorMap mBh,
                                                                         const __grid_constant__ CUtensorMap mBl,
                                                                         int M, int N, int K, float* __restrict__ C,
                                                                         int64_t ldc) {
  constexpr int STAGES = BLO ? 3 : 4;
  constexpr int STAGE = 2 * kATileBytes + (BLO ? 2 : 1) * kBTileBytes;
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t full[STAGES], empty[STAGES], acc_full, acc_empty;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int failed;
  uint8_t* base = raw + ((1024 - (tqtc::smem_u32(raw) & 1023)) & 1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles_n = (N + kGN - 1) / kGN;
  const int n_tiles = ((M + kGM - 1) / kGM) * tiles_n;
  const int KT = (K + kGK - 1) / kGK;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tqtc::mbar_init(&full[s], 1);
      tqtc::mbar_init(&empty[s], 1);
    }
    tqtc::mbar_init(&acc_full, 1);
    tqtc::mbar_init(&acc_empty, 128);
    failed = 0;
  }
  if (warp == 0) tqtc::tmem_alloc(&tmem_slot, kGAcc * kGN);
  tqtc::fence_before_sync();
  __syncthreads();
  tqtc::fence_after_sync();
  const uint32_t tmem = tmem_slot;
  auto stage_ptr = [&](int s) { return base + s * STAGE; };

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer: TMA loads of every tile's K tiles into the ring
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile / tiles_n) * kGM, n0 = (tile % tiles_n) * kGN;
        for (int kt = 0; kt < KT; ++kt, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES) ok = tqtc::mbar_wait(&empty[s], ((it / STAGES) - 1) & 1, kGWaitLimit);
          if (!ok || failed) {
            ok = false;
            break;
          }
          uint8_t* st = stage_ptr(s);
          tqtc::mbar_arrive_expect_tx(&full[s], STAGE);
          tqtc::tma_load_2d(st, &mAh, kt * kGK, m0, &full[s]);
          tqtc::tma_load_2d(st + kATileBytes, &mAl, kt * kGK, m0, &full[s]);
          tqtc::tma_load_2d(st + 2 * kATileBytes, &mBh, kt * kGK, n0, &full[s]);
          if constexpr (BLO) tqtc::tma_load_2d(st + 2 * kATileBytes + kBTileBytes, &mBl, kt * kGK, n0, &full[s]);
        }
      }
      if (!ok) failed = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer
      const uint32_t idesc = tqtc::idesc_bf16_f32(kGM, kGN);
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tc) {
        if (tc > 0) ok = tqtc::mbar_wait(&acc_empty, (tc - 1) & 1, kGWaitLimit);   // previous tile taken out
        if (!ok || failed) {
          ok = false;
          break;
        }
        tqtc::fence_after_sync();
        for (int kt = 0; kt < KT; ++kt, ++it) {
          const int s = it % STAGES;
          ok = tqtc::mbar_wait(&full[s], (it / STAGES) & 1, kGWaitLimit);
          if (!ok || failed) {
            ok = false;
            break;
          }
          tqtc::fence_after_sync();
          const uint32_t a_hi = tqtc::smem_u32(stage_ptr(s)), a_lo = a_hi + kATileBytes;
          const uint32_t b_hi = a_hi + 2 * kATileBytes, b_lo = b_hi + kBTileBytes;
          const uint32_t dacc = tmem + (kt % kGAcc) * kGN;
#pragma unroll
          for (int ks = 0; ks < kGK / 16; ++ks) {
            const bool acc = kt >= kGAcc || ks > 0;
            tqtc::mma_bf16_ss(dacc, tqtc::sw128_desc_kstep(a_hi, ks, kGM), tqtc::sw128_desc_kstep(b_hi, ks, kGN), idesc,
                              acc);
            if constexpr (BLO)
              tqtc::mma_bf16_ss(dacc, tqtc::sw128_desc_kstep(a_hi, ks, kGM), tqtc::sw128_desc_kstep(b_lo, ks, kGN),
                                idesc, true);
            tqtc::mma_bf16_ss(dacc, tqtc::sw128_desc_kstep(a_lo, ks, kGM), tqtc::sw128_desc_kstep(b_hi, ks, kGN), idesc,
                              true);
          }
          tqtc::mma_commit(&empty[s]);
        }
        if (!ok) break;
        tqtc::mma_commit(&acc_full);   // arrives once this tile's MMAs have completed
      }
      if (!ok) failed = 1;
    }
  } else {
    // ---- epilogue: thread = tensor-memory lane = row 32 (warp % 4) + lane of the tile
    const int r = 32 * (warp & 3) + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    const int n_acc = KT < kGAcc ? KT : kGAcc;
    int tc = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
      const int m0 = (tile / tiles_n) * kGM, n0 = (tile % tiles_n) * kGN;
      // warp-uniform: the tensor-memory loads below are .sync.aligned
      const bool ok = __all_sync(0xffffffffu, !failed && tqtc::mbar_wait(&acc_full, tc & 1, kGWaitLimit));
      tqtc::fence_after_sync();
      float v[kGN];
      if (ok) {
#pragma unroll
        for (int c = 0; c < kGN / 32; ++c) {
          float w[32];
          tqtc::tmem_ld32(tl + 32 * c, w);
#pragma unroll
          for (int q = 0; q < 32; ++q) v[32 * c + q] = w[q];
          for (int a = 1; a < n_acc; ++a) {
            tqtc::tmem_ld32(tl + a * kGN + 32 * c, w);
#pragma unroll
            for (int q = 0; q < 32; ++q) v[32 * c + q] += w[q];
          }
        }
      }
      tqtc::fence_before_sync();
      tqtc::mbar_arrive(&acc_empty);   // this lane's accumulators are in registers
      if (!ok) failed = 1;
      const int row = m0 + r;
      if (row < M) {
        float* dst = C + static_cast<int64_t>(row) * ldc + n0;
        if (n0 + kGN <= N && (ldc & 3) == 0) {
#pragma unroll
          for (int q = 0; q < kGN / 4; ++q)
            reinterpret_cast<float4*>(dst)[q] =
                ok ? make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]) : make_float4(NAN, NAN, NAN, NAN);
        } else {
#pragma unroll
          for (int q = 0; q < kGN; ++q)
            if (n0 + q < N) dst[q] = ok ? v[q] : NAN;
        }
      }
    }
  }
  __syncwarp();
  tqtc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tqtc::tmem_free(tmem, kGAcc * kGN);
}

// fp32 -> bf16 hi + lo pieces (round to nearest), row-major, one thread per 4 elements.
__global__ void split_bf16_kernel(const float* __restrict__ x, int64_t ldx, int64_t rows, int cols,
                                  __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo, int64_t ldo) {
  const int64_t q = cols / 4;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < rows * q;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / q;
    const int c = static_cast<int>(i % q) * 4;
    const float4 v = *reinterpret_cast<const float4*>(x + r * ldx + c);
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(v.x, v.y), h1 = __floats2bfloat162_rn(v.z, v.w);
    const __nv_bfloat162 l0 = __floats2bfloat162_rn(v.x - __low2float(h0), v.y - __high2float(h0));
    const __nv_bfloat162 l1 = __floats2bfloat162_rn(v.z - __low2float(h1), v.w - __high2float(h1));
    __nv_bfloat162* ph = reinterpret_cast<__nv_bfloat162*>(hi + r * ldo + c);
    __nv_bfloat162* pl = reinterpret_cast<__nv_bfloat162*>(lo + r * ldo + c);
    ph[0] = h0;
    ph[1] = h1;
    pl[0] = l0;
    pl[1] = l1;
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// Tensor map of a row-major bf16 matrix [rows][cols] (ld elements per row)
// read in boxes of 64 columns x box_rows rows with a 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  return tq::make_tmap_2d(map, ptr, 2, rows, cols, ld, kGK, box_rows);
}

}  // namespace

namespace tq {

bool make_tmap_2d(CUtensorMap* map, const void* ptr, int elem_bytes, int64_t rows, int64_t cols, int64_t ld,
                  int box_cols, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn || (elem_bytes != 2 && elem_bytes != 4)) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * elem_bytes};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  return fn(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int split_bf16(const float* x, int64_t ldx, int64_t rows, int cols, uint16_t* hi, uint16_t* lo, int64_t ldo,
               cudaStream_t s) {
  if (rows <= 0) return TQ_OK;
  if ((cols & 3) || (ldx & 3) || (ldo & 3)) return TQ_EINVAL;
  const int64_t items = rows * (cols / 4);
  const int blocks = static_cast<int>(items / 256 + 1 < 148 * 16 ? items / 256 + 1 : 148 * 16);
  split_bf16_kernel<<<blocks, 256, 0, s>>>(x, ldx, rows, cols, reinterpret_cast<__nv_bfloat16*>(hi),
                                           reinterpret_cast<__nv_bfloat16*>(lo), ldo);
  return launch_status();
}

int tc_gemm_split(int M, int N, int K, const uint16_t* ah, const uint16_t* al, int64_t lda, const uint16_t* bh,
                  const uint16_t* bl, int64_t ldb, float* C, int64_t ldc, cudaStream_t s) {
  if (M <= 0 || N <= 0) return TQ_OK;
  if (K <= 0 || (lda & 7) || (ldb & 7) || !aligned16(ah) || !aligned16(al) || !aligned16(bh) ||
      (bl && !aligned16(bl)))
    return TQ_EINVAL;
  alignas(64) CUtensorMap mah, mal, mbh, mbl;
  if (!make_map(&mah, ah, M, K, lda, kGM) || !make_map(&mal, al, M, K, lda, kGM) ||
      !make_map(&mbh, bh, N, K, ldb, kGN) || !make_map(&mbl, bl ? bl : bh, N, K, ldb, kGN))
    return TQ_ECUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t n_tiles = static_cast<int64_t>((M + kGM - 1) / kGM) * ((N + kGN - 1) / kGN);
  const dim3 grid(static_cast<unsigned>(n_tiles < sms ? n_tiles : sms));
  if (bl) {
    const size_t smem = 3 * (2 * kATileBytes + 2 * kBTileBytes) + 1024;
    if (cudaFuncSetAttribute(tc_gemm_persistent_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return TQ_ECUDA;
    tc_gemm_persistent_kernel<true><<<grid, kPThreads, smem, s>>>(mah, mal, mbh, mbl, M, N, K, C, ldc);
  } else {
    const size_t smem = 4 * (2 * kATileBytes + kBTileBytes) + 1024;
    if (cudaFuncSetAttribute(tc_gemm_persistent_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return TQ_ECUDA;
    tc_gemm_persistent_kernel<false><<<grid, kPThreads, smem, s>>>(mah, mal, mbh, mbl, M, N, K, C, ldc);
  }
  return launch_status();
}

}  // namespace tq
