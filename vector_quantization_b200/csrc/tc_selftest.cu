// Device self-test of the tensor-core (tcgen05) forms the kernels rely on:
// one 128 x 128 x 128 bf16 product and two 128 x 64 x 64 products (B K-major,
// and B MN-major as the value operand of the encoder attention kernel), with
// exactly representable small-integer operands in the 128-byte swizzled
// shared-memory layouts, computed into tensor memory and read back, compared
// element by element with the exact integer results on the host.
#include <cstdlib>
#include <vector>

#include <cuda_bf16.h>

#include "tcgen05.cuh"
#include "tq_internal.h"

namespace {

constexpr int kN = 128;
constexpr int kWaitLimit = 1 << 17;   // polls of about 9 us each: a wait gives up after about a second

__device__ __host__ inline int sel_a(int r, int k) { return (r * 7 + k * 3) % 11 - 5; }
__device__ __host__ inline int sel_b(int n, int k) { return (n * 5 + k) % 9 - 4; }

__global__ void __launch_bounds__(128) tc_selftest_kernel(float* __restrict__ out, int* __restrict__ status) {
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t mbar;
  __shared__ uint32_t tmem_slot;
  uint8_t* base = raw + ((1024 - (tqtc::smem_u32(raw) & 1023)) & 1023);
  uint8_t* A = base;
  uint8_t* B = base + kN * kN * 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < kN * kN; i += blockDim.x) {
    const int r = i / kN, k = i % kN;
    *reinterpret_cast<__nv_bfloat16*>(A + tqtc::sw128_offset(r, k, kN)) = __float2bfloat16_rn(static_cast<float>(sel_a(r, k)));
    *reinterpret_cast<__nv_bfloat16*>(B + tqtc::sw128_offset(r, k, kN)) = __float2bfloat16_rn(static_cast<float>(sel_b(r, k)));
  }
  if (tid == 0) tqtc::mbar_init(&mbar, 1);
  if (warp == 0) tqtc::tmem_alloc(&tmem_slot, kN);
  tqtc::fence_smem_to_async();
  tqtc::fence_before_sync();
  __syncthreads();
  tqtc::fence_after_sync();
  const uint32_t tmem = tmem_slot;
  if (tid == 0) {
    const uint32_t idesc = tqtc::idesc_bf16_f32(kN, kN);
    for (int ks = 0; ks < kN / 16; ++ks)
      tqtc::mma_bf16_ss(tmem, tqtc::sw128_desc_kstep(tqtc::smem_u32(A), ks, kN),
                        tqtc::sw128_desc_kstep(tqtc::smem_u32(B), ks, kN), idesc, ks > 0);
    tqtc::mma_commit(&mbar);
  }
  const bool ok = tqtc::mbar_wait(&mbar, 0, kWaitLimit);
  if (!ok && lane == 0) atomicExch(status, 1);
  tqtc::fence_after_sync();
  if (ok) {
    const int row = warp * 32 + lane;
    for (int c0 = 0; c0 < kN; c0 += 32) {
      float v[32];
      tqtc::tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
      for (int j = 0; j < 32; ++j) out[row * kN + c0 + j] = v[j];
    }
  }
  tqtc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tqtc::tmem_free(tmem, kN);
}

// 128 x 64 x 64: D[m][n] = sum_k A[m][k] B[k][n], B stored K-major (row n,
// column k) or MN-major (row k holding the 64 n of that k).
constexpr int kM2 = 128, kN2 = 64, kK2 = 64;
__device__ __host__ inline int sel_a2(int m, int k) { return (m * 7 + k * 3) % 11 - 5; }
__device__ __host__ inline int sel_b2(int k, int n) { return (n * 5 + k * 13) % 9 - 4; }

__global__ void __launch_bounds__(128) tc_selftest_n64_kernel(int mn_major, float* __restrict__ out,
                                                              int* __restrict__ status) {
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t mbar;
  __shared__ uint32_t tmem_slot;
  uint8_t* base = raw + ((1024 - (tqtc::smem_u32(raw) & 1023)) & 1023);
  uint8_t* A = base;
  uint8_t* B = base + kM2 * kK2 * 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < kM2 * kK2; i += blockDim.x) {
    const int m = i / kK2, k = i % kK2;
    *reinterpret_cast<__nv_bfloat16*>(A + tqtc::sw128_offset(m, k, kM2)) =
        __float2bfloat16_rn(static_cast<float>(sel_a2(m, k)));
  }
  for (int i = tid; i < kK2 * kN2; i += blockDim.x) {
    const int k = i / kN2, n = i % kN2;
    const uint32_t off = mn_major ? static_cast<uint32_t>((k >> 3) * 1024 + (k & 7) * 128 +
                                                          (((n >> 3) ^ (k & 7)) << 4) + ((n & 7) << 1))
                                  : tqtc::sw128_offset(n, k, kN2);
    *reinterpret_cast<__nv_bfloat16*>(B + off) = __float2bfloat16_rn(static_cast<float>(sel_b2(k, n)));
  }
  if (tid == 0) tqtc::mbar_init(&mbar, 1);
  if (warp == 0) tqtc::tmem_alloc(&tmem_slot, kN2);
  tqtc::fence_smem_to_async();
  tqtc::fence_before_sync();
  __syncthreads();
  tqtc::fence_after_sync();
  const uint32_t tmem = tmem_slot;
  if (tid == 0) {
    const uint32_t idesc = tqtc::idesc_bf16_f32(kM2, kN2) | (mn_major ? tqtc::kIdescBMajorMN : 0u);
    for (int ks = 0; ks < kK2 / 16; ++ks) {
      const uint64_t bd = mn_major ? tqtc::sw128_desc_mn(tqtc::smem_u32(B) + ks * 2048)
                                   : tqtc::sw128_desc_kstep(tqtc::smem_u32(B), ks, kN2);
      tqtc::mma_bf16_ss(tmem, tqtc::sw128_desc_kstep(tqtc::smem_u32(A), ks, kM2), bd, idesc, ks > 0);
    }
    tqtc::mma_commit(&mbar);
  }
  const bool ok = tqtc::mbar_wait(&mbar, 0, kWaitLimit);
  if (!ok && lane == 0) atomicExch(status, 1);
  tqtc::fence_after_sync();
  if (ok) {
    const int row = warp * 32 + lane;
    for (int c0 = 0; c0 < kN2; c0 += 32) {
      float v[32];
      tqtc::tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
      for (int j = 0; j < 32; ++j) out[row * kN2 + c0 + j] = v[j];
    }
  }
  tqtc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tqtc::tmem_free(tmem, kN2);
}

// Bounded-wait check: thread 0 inits an mbarrier expecting one arrival.
// With `arrive` it arrives first and the wait must see the phase complete;
// without, nothing ever completes the phase and the wait must give up after
// `limit` polls.  status[0] = 1 if the wait saw completion, 0 if it gave up.
__global__ void wait_selftest_kernel(int arrive, int limit, int* __restrict__ status) {
  __shared__ uint64_t mbar;
  if (threadIdx.x != 0) return;
  tqtc::mbar_init(&mbar, 1);
  if (arrive) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(tqtc::smem_u32(&mbar)) : "memory");
  status[0] = tqtc::mbar_wait(&mbar, 0, limit) ? 1 : 0;
}

}  // namespace

extern "C" int tq_wait_selftest(int arrive, int* completed) {
  if (!completed) return TQ_EINVAL;
  *completed = -1;
  int* d_status = nullptr;
  if (cudaMalloc(&d_status, sizeof(int)) != cudaSuccess) return TQ_ENOMEM;
  int st = TQ_OK;
  int h = -1;
  if (cudaMemset(d_status, 0xFF, sizeof(int)) != cudaSuccess) {
    st = TQ_ECUDA;
  } else {
    wait_selftest_kernel<<<1, 32>>>(arrive ? 1 : 0, 1 << 16, d_status);
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(&h, d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
      st = TQ_ECUDA;
    else
      *completed = h;
  }
  cudaFree(d_status);
  return st;
}

extern "C" int tq_tensor_core_selftest(int64_t* mismatches) {
  if (!mismatches) return TQ_EINVAL;
  *mismatches = -1;
  float* d_out = nullptr;
  int* d_status = nullptr;
  if (cudaMalloc(&d_out, sizeof(float) * kN * kN) != cudaSuccess) return TQ_ENOMEM;
  if (cudaMalloc(&d_status, sizeof(int)) != cudaSuccess) {
    cudaFree(d_out);
    return TQ_ENOMEM;
  }
  int st = TQ_OK;
  const int smem = 2 * kN * kN * 2 + 1024;
  if (cudaMemset(d_status, 0, sizeof(int)) != cudaSuccess || cudaMemset(d_out, 0xFF, sizeof(float) * kN * kN) != cudaSuccess ||
      cudaFuncSetAttribute(tc_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    st = TQ_ECUDA;
  } else {
    tc_selftest_kernel<<<1, 128, smem>>>(d_out, d_status);
    std::vector<float> out(kN * kN);
    int status = 0;
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(out.data(), d_out, sizeof(float) * kN * kN, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(&status, d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
      st = TQ_ECUDA;
    } else {
      int64_t bad = status ? kN * kN : 0;
      for (int m = 0; m < kN && !status; ++m)
        for (int n = 0; n < kN; ++n) {
          long ref = 0;
          for (int k = 0; k < kN; ++k) ref += static_cast<long>(sel_a(m, k)) * sel_b(n, k);
          if (out[m * kN + n] != static_cast<float>(ref)) ++bad;
        }
      *mismatches = bad;
    }
  }
  // the two 128 x 64 x 64 forms
  const int smem2 = kM2 * kK2 * 2 + kK2 * kN2 * 2 + 1024;
  if (st == TQ_OK &&
      cudaFuncSetAttribute(tc_selftest_n64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2) != cudaSuccess)
    st = TQ_ECUDA;
  for (int mn = 0; mn < 2 && st == TQ_OK; ++mn) {
    std::vector<float> out(kM2 * kN2);
    int status = 0;
    if (cudaMemset(d_status, 0, sizeof(int)) != cudaSuccess ||
        cudaMemset(d_out, 0xFF, sizeof(float) * kM2 * kN2) != cudaSuccess) {
      st = TQ_ECUDA;
      break;
    }
    tc_selftest_n64_kernel<<<1, 128, smem2>>>(mn, d_out, d_status);
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(out.data(), d_out, sizeof(float) * kM2 * kN2, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(&status, d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
      st = TQ_ECUDA;
      break;
    }
    int64_t bad = status ? kM2 * kN2 : 0;
    for (int m = 0; m < kM2 && !status; ++m)
      for (int n = 0; n < kN2; ++n) {
        long ref = 0;
        for (int k = 0; k < kK2; ++k) ref += static_cast<long>(sel_a2(m, k)) * sel_b2(k, n);
        if (out[m * kN2 + n] != static_cast<float>(ref)) ++bad;
      }
    *mismatches += bad;
  }
  cudaFree(d_out);
  cudaFree(d_status);
  return st;
}
