// Device helpers shared by the attention kernels: async copies, warp-level
// MMA wrappers, and the construction of exact tensor-core operands from
// packed code / sign bit-planes.
//
// A b-bit Lloyd-Max code is used in Walsh form,
//   c[idx] = sum_p w_p s_p(idx),  s_p a product of the code's bits as +-1
// (b = 1: s_0; b = 2: s_1, s_0; b = 3: s_2, s_1, s_0, s_0 s_1 s_2), so every
// contraction with dequantized keys or values becomes a sum of contractions
// with exact +-1 matrices built directly from the packed bits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace tqdev {

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, int src_bytes) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gsrc), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Transposing loads of four (two) 8 x 8 matrices of 16-bit elements from
// shared memory; lane l supplies the 16-byte-aligned address of row l % 8 of
// matrix l / 8, and register m of lane (g = l / 4, t = l % 4) receives
// elements (row 2t, column g) and (row 2t + 1, column g) of matrix m.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t& r0, uint32_t& r1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"(addr)
               : "memory");
}

// D += A B, m16n8k16, bf16 operands, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A B, m16n8k16, fp16 operands, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A B, m16n8k32, A unsigned 8-bit, B signed 8-bit, int32 accumulate
// (exact).  Fragments: a0/a1 rows g/g+8 at K 4t..4t+3, a2/a3 the same rows at
// K 16+4t..; b0 K 4t.., b1 K 16+4t.. of column g; c0,c1 row g columns 2t,
// 2t+1 and c2,c3 row g+8 (g = lane / 4, t = lane % 4).
__device__ __forceinline__ void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Integer accumulators started at kBiasedZero hold 1.5 * 2^23 + x as a float
// bit pattern while |x| < 2^22, so the float value of x is one subtraction.
constexpr int kBiasedZero = 0x4B400000;
__device__ __forceinline__ float biased_to_float(int b) { return __int_as_float(b) - 12582912.0f; }

// Two biased digit sums at once (fp32x2: the same rounding as two calls).
__device__ __forceinline__ float2 biased_to_float2(int a, int b) {
  return __fadd2_rn(make_float2(__int_as_float(a), __int_as_float(b)), make_float2(-12582912.0f, -12582912.0f));
}

// digits_to_float of two rows at once: digit k of row 0 in a[k], of row 1 in b[k].
__device__ __forceinline__ float2 digits_to_float2(const int (&a)[4], const int (&b)[4]) {
  const float2 s = make_float2(256.f, 256.f);
  float2 f = biased_to_float2(a[3], b[3]);
  f = __ffma2_rn(f, s, biased_to_float2(a[2], b[2]));
  f = __ffma2_rn(f, s, biased_to_float2(a[1], b[1]));
  return __ffma2_rn(f, s, biased_to_float2(a[0], b[0]));
}

// d0 + 2^8 d1 + 2^16 d2 + 2^24 d3 in fp32 from four biased digit sums.
__device__ __forceinline__ float digits_to_float(int b0, int b1, int b2, int b3) {
  float f = biased_to_float(b3);
  f = fmaf(f, 256.f, biased_to_float(b2));
  f = fmaf(f, 256.f, biased_to_float(b1));
  return fmaf(f, 256.f, biased_to_float(b0));
}

// Two bf16 values +-1 from bits x (low half) and x+16 (high half) of w:
// bit = 1 -> +1.0, bit = 0 -> -1.0 (one shift and one LOP3).
__device__ __forceinline__ uint32_t pm1_pair(uint32_t w, int x) {
  const uint32_t t = w << (15 - x);
  return (~t & 0x80008000u) | 0x3F803F80u;
}

// Bits j and j+16 of a plane word as a pair of fp16 values in ONE LOP3.
// The kept bit sits at half-word position p = j + 8 (taken from w << 8) for
// j < 8, or p = j for j >= 8, inside a fixed fp16 pattern pos_base_h(p):
// positions 8-9 are mantissa bits of 1.0, 10-14 exponent bits, 15 the sign.
// The pair element is then v0(p) (bit 0) or v1(p) (bit 1), both exact, so
// with s = 2 bit - 1 it equals mu_p + sigma_p s.  Callers divide sigma_p
// out of the other operand and subtract sum_k mu_k B_k once per row/column.
//
// Every pattern except p = 14 is 1.0 with bit p cleared, so the pair is a
// bit-select of w under the mask and the register constant `one` = 1.0 in
// both halves: (w & M) | (one & ~M), one LOP3 with the mask as immediate
// and a single register shared by all slots (p = 14 is w & M).  `one` must
// reach the kernel as a runtime value (a kernel parameter), so the compiler
// cannot fold it into a second immediate.
__host__ __device__ constexpr uint32_t pos_base_h(int p) {
  return p == 8 ? 0x3C00u : p == 9 ? 0x3C00u : p == 10 ? 0x3800u : p == 11 ? 0x3400u
       : p == 12 ? 0x2C00u : p == 13 ? 0x1C00u : p == 14 ? 0x0000u : 0x3C00u;
}
constexpr uint32_t kOneH2 = 0x3C003C00u;   // fp16 1.0 in both halves
constexpr uint32_t kOneB2 = 0x3F803F80u;   // bf16 1.0 in both halves

__device__ __forceinline__ uint32_t bit_select(uint32_t w, int p, uint32_t one) {
  const uint32_t mask = (1u << p) | (1u << (p + 16));
  uint32_t d;
  if (p == 14) asm("lop3.b32 %0, %1, %2, %3, 0xC0;" : "=r"(d) : "r"(w), "r"(mask), "r"(one));
  else asm("lop3.b32 %0, %1, %2, %3, 0xE2;" : "=r"(d) : "r"(w), "r"(mask), "r"(one));
  return d;
}
// one_h must hold kOneH2.
__device__ __forceinline__ uint32_t bit_pair_h(uint32_t w, uint32_t w_shl8, int j, uint32_t one_h) {
  return bit_select(j < 8 ? w_shl8 : w, j < 8 ? j + 8 : j, one_h);
}
__host__ __device__ constexpr float pos_v0_h(int p) {
  return p == 8 ? 1.f : p == 9 ? 1.f : p == 10 ? 0.5f : p == 11 ? 0.25f : p == 12 ? 0.0625f
       : p == 13 ? 0.00390625f : p == 14 ? 0.f : 1.f;
}
__host__ __device__ constexpr float pos_v1_h(int p) {
  return p == 8 ? 1.25f : p == 9 ? 1.5f : p == 14 ? 2.f : p == 15 ? -1.f : 1.f;
}
// Position of pair slot j (see bit_pair_h).
__host__ __device__ constexpr int slot_pos(int j) { return j < 8 ? j + 8 : j; }

// The same construction for bf16 operands: kept bit at position p = 8..14
// (bf16 exponent bits) or 15 (sign) inside the pattern pos_base_b(p), again
// 1.0 with bit p cleared except p = 14; one_b must hold kOneB2.
__host__ __device__ constexpr uint32_t pos_base_b(int p) {
  return p == 8 ? 0x3E80u : p == 9 ? 0x3D80u : p == 10 ? 0x3B80u : p == 11 ? 0x3780u
       : p == 12 ? 0x2F80u : p == 13 ? 0x1F80u : p == 14 ? 0x0000u : 0x3F80u;
}
__device__ __forceinline__ uint32_t bit_pair_b(uint32_t w, uint32_t w_shl8, int j, uint32_t one_b) {
  return bit_select(j < 8 ? w_shl8 : w, j < 8 ? j + 8 : j, one_b);
}
__host__ __device__ constexpr float pos_v0_b(int p) {
  return p == 8 ? 0.25f : p == 9 ? 0.0625f : p == 10 ? 0.00390625f : p == 11 ? 1.52587890625e-05f
       : p == 12 ? 2.3283064365386963e-10f : p == 13 ? 5.421010862427522e-20f : p == 14 ? 0.f : 1.f;
}
__host__ __device__ constexpr float pos_v1_b(int p) { return p == 14 ? 2.f : p == 15 ? -1.f : 1.f; }

constexpr bool bases_are_one_minus_bit() {
  for (int p = 8; p < 16; ++p) {
    if (p == 14) {
      if (pos_base_h(p) != 0 || pos_base_b(p) != 0) return false;
    } else if (pos_base_h(p) != (0x3C00u & ~(1u << p)) || pos_base_b(p) != (0x3F80u & ~(1u << p))) {
      return false;
    }
  }
  return true;
}
static_assert(bases_are_one_minus_bit(), "bit_select relies on the patterns being 1.0 with bit p cleared");

// fp32 bits rounded to the nearest bf16 (ties away from zero), low half zero.
__device__ __forceinline__ uint32_t bf16_round_bits(float w) { return (__float_as_uint(w) + 0x8000u) & 0xFFFF0000u; }

// Power-of-two factor bringing max |x| to [2^13, 2^14) (1 for x = 0), so
// that fp16 pieces of scaled values never overflow.
__device__ __forceinline__ float fp16_range_scale(float max_abs) {
  if (!(max_abs > 0.f) || !isfinite(max_abs)) return 1.f;
  int e;
  frexpf(max_abs, &e);           // max_abs in [2^(e-1), 2^e)
  return ldexpf(1.f, 14 - e);
}

// 2^x by the hardware approximation (PTX ex2.approx: relative error near
// 2^-22, subnormal results flushed to zero, 2^-inf = +0), for softmax
// weights, which need no more.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(lo))) |
         (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(hi))) << 16);
}

template <int BITS>
struct Planes {
  static constexpr int P = BITS == 1 ? 1 : (BITS == 2 ? 2 : 4);
  // Walsh planes from raw bit-plane words (same element layout in all words).
  __device__ static __forceinline__ void make(const uint32_t (&raw)[BITS], uint32_t (&out)[P]) {
    if constexpr (BITS == 1) {
      out[0] = raw[0];
    } else if constexpr (BITS == 2) {
      out[0] = raw[1];
      out[1] = raw[0];
    } else {
      out[0] = raw[2];
      out[1] = raw[1];
      out[2] = raw[0];
      out[3] = raw[0] ^ raw[1] ^ raw[2];  // s0 s1 s2 = +1 iff an odd number of bits are 1
    }
  }
};

}  // namespace tqdev
