// Private declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "../../include/tq.h"

// Codec handle.  Host copies keep what the host-side launch code needs;
// device copies are what the kernels read.  Immutable after build.
struct tq_rotation {
  int device = 0;
  int d = 0, m = 0, bits = 0, kind = 0;
  // Residual correction: TQ_RES_QJL (sign(S r), ||r||, constant sqrt(pi/2)/m)
  // or TQ_RES_SIGN (sign(r), mean |r_i|, constant 1: S is the identity).
  int residual = 0;
  double res_const = 0.0;
  double rope_base = 0.0;
  int64_t rope_max_pos = 0;
  int rope_hi_rows = 0;                 // rows of the coarse RoPE table
  // RoPE frequencies theta_i = base^(-2i/d), i < d/2, as float hi + lo pieces
  // (theta_i - hi - lo within about 2^-48 theta_i)
  float rope_th_hi[64] = {}, rope_th_lo[64] = {};

  std::vector<double> levels;           // [2^bits] ascending
  std::vector<double> thresholds;       // [2^bits - 1]
  std::vector<float> signs;             // [d] +-1 (Hadamard kind)
  // Walsh form of the codebook: level(idx) = sum_p walsh[p] * s_p(idx),
  // s_p the +-1 value of the p-th plane product (see plane_products()).
  double walsh[4] = {0, 0, 0, 0};
  int n_planes = 0;                     // 1, 2 or 4 for bits 1, 2, 3

  // device
  float* d_levels = nullptr;            // [2^bits]
  float* d_thresholds = nullptr;        // [2^bits - 1]
  float* d_signs = nullptr;             // [d] +-1 (Hadamard kind)
  float* d_pi = nullptr;                // [d*d] row-major (dense kind)
  float* d_s = nullptr;                 // [m*d] row-major S (bf16-exact values)
  float* d_st = nullptr;                // [d*m] S transposed
  // S as bf16 in the tensor-core operand layout (K-major, 128-byte swizzle,
  // rows = sketch index, K = coordinate); Hadamard kind only.
  uint16_t* d_s_op = nullptr;
  // H D (the unnormalised Hadamard times the sign diagonal, entries +-1) in
  // the same operand layout, rows = output coordinate, as fp16 and as bf16
  // bits; Hadamard kind, d = 64 and 128.
  uint16_t* d_hd_f16 = nullptr;
  uint16_t* d_hd_bf16 = nullptr;
  // Hadamard kind, d = 64: the output transform of the tensor-core encoder
  // attention, out = D H (O_code + qjl S^T O_z) / sqrt(d), as three bf16
  // operands [64 output coordinates x 64 slots] in the same layout, columns
  // in the kernel's slot order (slot k = coordinate 32 (k / 32) + (k / 2) % 16
  // + 16 (k % 2)): D H / 8 (exact), then qjl D H S^T / 8 as hi and lo pieces.
  uint16_t* d_enc_epi = nullptr;
  // Dense kind: Pi as bf16 hi + lo pieces and S as bf16, row-major, for the
  // split tensor-core contractions.
  uint16_t* d_pi_hi = nullptr;
  uint16_t* d_pi_lo = nullptr;
  uint16_t* d_s_bf16 = nullptr;
  float2* d_rope_hi = nullptr;          // [rope_hi_rows][d/2] (cos, sin) of h*1024*theta_i
  float2* d_rope_lo = nullptr;          // [1024][d/2]           (cos, sin) of l*theta_i
};

// Number of low position bits resolved by the fine RoPE table.
constexpr int kRopeLoBits = 10;
constexpr int kRopeLoRows = 1 << kRopeLoBits;

// sqrt(pi/2): the QJL estimator constant (divided by m at use).
constexpr double kQjlConst = 1.2533141373155002512078826424055226;

namespace tq {

// Checks that the current device is the handle's device.
bool on_handle_device(const tq_rotation* h);

// Uniform launch-error check after a kernel launch.
inline int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Tensor map (2-D, 128-byte swizzle, zero fill past the edges) of a row-major
// matrix [rows][cols] of bf16 (elem_bytes 2) or fp32 (4) elements with ld
// elements per row, read in boxes of box_cols x box_rows; false when the
// driver entry point is missing or the arguments break the TMA rules (base
// 16-byte aligned, ld * elem_bytes a multiple of 16).
bool make_tmap_2d(CUtensorMap* map, const void* ptr, int elem_bytes, int64_t rows, int64_t cols, int64_t ld,
                  int box_cols, int box_rows);

// fp32 -> bf16 hi + lo pieces of a row-major matrix (cols % 4 == 0).
int split_bf16(const float* x, int64_t ldx, int64_t rows, int cols, uint16_t* hi, uint16_t* lo, int64_t ldo,
               cudaStream_t s);
// C[M][N] = A[M][K] B[N][K]^T from bf16 pieces on the tensor core
// (A_hi B_hi + A_hi B_lo + A_lo B_hi; bl == nullptr drops the B_lo term).
int tc_gemm_split(int M, int N, int K, const uint16_t* ah, const uint16_t* al, int64_t lda, const uint16_t* bh,
                  const uint16_t* bl, int64_t ldb, float* C, int64_t ldc, cudaStream_t s);

}  // namespace tq
