// Bidirectional encoder attention over a packed K/V cache.
//
// Every query of a head attends to all T packed keys of its KV head, with
// the same estimator as decode ([TurboQuant] "QJL": score = <q~, ||k|| c[idx]>
// + ||r|| sqrt(pi/2)/m <S q~, sign(S r)>, q~ = Pi RoPE(q)) and the values
// dequantized after the weighted sum ([TurboESM] §2.E: dequantization,
// residual correction, inverse rotation Pi^T and an online softmax in one
// pass).  Queries sit at positions q_pos_offset + s.
//
// Two launches: a q-prep kernel (one warp per query: RoPE, fast
// Walsh-Hadamard rotation, S q~) and an attention kernel.  For d = 64 with 1-
// or 2-bit codes that is the tensor-core kernel further down (tcgen05,
// accumulators in tensor memory).  Otherwise it is the kernel below,
// flash-attention shaped on mma.sync m16n8k16 (bf16 in, fp32
// accumulate): a warp owns 8 queries, whose hi and lo bf16 pieces form the 16
// rows of the A operand, so both pieces of one query land in the same thread
// and are summed there.  Keys enter as the B operand straight from their bit
// planes (one LOP3 per register, the code bit in a bf16 exponent or sign
// field - see decode.cu), probabilities are reused in registers as the A
// operand of the value product, and values enter as +-1 bit-plane B operands.
// Key/value chunks are staged in shared memory with cp.async and shared by
// the 8 warps of a CTA; the epilogue applies S^T, Pi^T and 1/l per query.
#include <cuda_bf16.h>

#include <cmath>

#include "bitplane.cuh"
#include "tcgen05.cuh"
#include "tq_internal.h"

namespace {

using namespace tqdev;

constexpr int kWarps = 4;          // warps per CTA, 8 queries each (3 CTAs per SM at d = 64)
constexpr int kQPerWarp = 8;
constexpr int kChunk = 128;        // keys staged per shared-memory chunk
constexpr float kLazyRescale = 8.0f;

struct EncParams {
  const float* qprep;      // [B*Hq][S][2][D]: q~ and S q~
  const uint8_t* k_codes;
  const uint8_t* k_signs;
  const float2* k_norms;
  const uint8_t* v_codes;
  const uint8_t* v_signs;
  const float2* v_norms;
  int64_t cache_stride;
  int64_t T;
  int S, Hq, G;
  float score_scale;       // scale * log2(e)
  float qjl_k, qjl_v;      // sqrt(pi/2) / m of the K and V handles
  float walsh_k[4];
  float walsh_v[4];
  uint32_t one_h, one_b;   // kOneH2 / kOneB2, passed at run time (see bit_select)
  const float* v_s;        // [D][D] S_V row-major
  const float* v_signs_d;  // [D] Hadamard signs of the V handle
  const uint16_t* epi;     // output-transform operands of the V handle (d = 64; tensor-core kernel)
  float* out;              // [B*Hq][S][D]
};

// q-prep: one warp per query; lane l holds dims l + 32 j.
template <int D, typename T>
__global__ void __launch_bounds__(256) encoder_qprep_kernel(const T* __restrict__ q, int64_t n_queries, int S,
                                                            int64_t q_pos_offset, const float* __restrict__ dsigns,
                                                            const float* __restrict__ st, const float2* __restrict__ rope_hi,
                                                            const float2* __restrict__ rope_lo, int64_t rope_max_pos,
                                                            int rope, float* __restrict__ out) {
  constexpr int NJ = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t qi = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (qi >= n_queries) return;
  float v[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    if constexpr (sizeof(T) == 4) v[j] = q[qi * D + lane + 32 * j];
    else v[j] = __bfloat162float(q[qi * D + lane + 32 * j]);
  }
  if (rope) {
    const int64_t pos = q_pos_offset + qi % S;
    if (pos < 0 || pos >= rope_max_pos) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) v[j] = __int_as_float(0x7fc00000);
    } else {
      const float2* hi = rope_hi + (pos >> kRopeLoBits) * (D / 2);
      const float2* lo = rope_lo + (pos & (kRopeLoRows - 1)) * (D / 2);
#pragma unroll
      for (int j = 0; j < NJ / 2; ++j) {
        const int i = lane + 32 * j;
        const float2 a = hi[i], b = lo[i];
        const float c = a.x * b.x - a.y * b.y, s = a.y * b.x + a.x * b.y;
        const float x1 = v[j], x2 = v[j + NJ / 2];
        v[j] = x1 * c - x2 * s;
        v[j + NJ / 2] = x2 * c + x1 * s;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < NJ; ++j) v[j] *= dsigns[lane + 32 * j];
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const bool upper = (lane >> s) & 1;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const float o = __shfl_xor_sync(0xffffffffu, v[j], 1 << s);
      v[j] = upper ? o - v[j] : v[j] + o;
    }
  }
#pragma unroll
  for (int b = 1; b < NJ; b <<= 1)
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      if (j & b) continue;
      const float a0 = v[j], a1 = v[j | b];
      v[j] = a0 + a1;
      v[j | b] = a0 - a1;
    }
  const float inv = rsqrtf(static_cast<float>(D));
  float* o = out + qi * 2 * D;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    v[j] *= inv;
    o[lane + 32 * j] = v[j];
  }
  // s = S q~: s_r = sum_i S[r][i] q~_i, rows r = lane + 32 jj
  float acc[NJ];
#pragma unroll
  for (int jj = 0; jj < NJ; ++jj) acc[jj] = 0.f;
#pragma unroll
  for (int j = 0; j < NJ; ++j)
#pragma unroll 8
    for (int l = 0; l < 32; ++l) {
      const int i = l + 32 * j;
      const float qi_v = __shfl_sync(0xffffffffu, v[j], l);
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) acc[jj] = fmaf(st[i * D + lane + 32 * jj], qi_v, acc[jj]);
    }
#pragma unroll
  for (int jj = 0; jj < NJ; ++jj) o[D + lane + 32 * jj] = acc[jj];
}

template <int D, int BITS>
__global__ void __launch_bounds__(kWarps * 32, D == 64 ? 3 : 1) encoder_attention_kernel(EncParams p) {
  constexpr int P = Planes<BITS>::P;
  constexpr int CB = BITS * D / 8, SB = D / 8;
  constexpr int KB = D / 16;             // k-blocks of the score MMA
  constexpr int DT = D / 8;              // n-tiles of dims in the value MMA
  constexpr int HALF = kChunk * (CB + SB + 8);
  constexpr int STAGE = 2 * HALF;
  constexpr int NCHUNK16 = STAGE / 16;
  extern __shared__ __align__(16) uint8_t smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int bq = blockIdx.y;                       // b * Hq + h
  const int b = bq / p.Hq, h = bq % p.Hq;
  const int bh = b * (p.Hq / p.G) + h / p.G;
  const int q0 = blockIdx.x * (kWarps * kQPerWarp) + warp * kQPerWarp;
  const int64_t seq = static_cast<int64_t>(bh) * p.cache_stride;
  const int n_chunks = static_cast<int>((p.T + kChunk - 1) / kChunk);

  // ---- query A fragments: fp16 hi (rows gid) / lo (rows gid + 8) pieces of
  // x / sigma_p scaled by a per-query power of two into fp16 range ---------
  uint32_t qa[2][KB][4];
  float2 kconst[2];          // (sum_k mu_k A_k, 1 / scale) for query gid
  {
    const int qrow = min(q0 + gid, p.S - 1);
    const float* src = p.qprep + (static_cast<int64_t>(bq) * p.S + qrow) * 2 * D;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      float xs[D / 8][2];
      float mx = 0.f;
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        // pair slot j of this lane's key word holds dims tig*D/4 + j and + D/8
        const int pp = slot_pos(j);
        const float sigma = 0.5f * (pos_v1_h(pp) - pos_v0_h(pp));
        xs[j][0] = src[t * D + tig * (D / 4) + j] / sigma;
        xs[j][1] = src[t * D + tig * (D / 4) + j + D / 8] / sigma;
        mx = fmaxf(mx, fmaxf(fabsf(xs[j][0]), fabsf(xs[j][1])));
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float lam = fp16_range_scale(mx);
      float csum = 0.f;
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        const int pp = slot_pos(j);
        const float mu = 0.5f * (pos_v0_h(pp) + pos_v1_h(pp));
        const float x0 = xs[j][0] * lam, x1 = xs[j][1] * lam;
        const float h0 = __half2float(__float2half_rn(x0)), h1 = __half2float(__float2half_rn(x1));
        const float l0 = __half2float(__float2half_rn(x0 - h0));
        const float l1 = __half2float(__float2half_rn(x1 - h1));
        const int kb = j >> 1, r = j & 1;
        qa[t][kb][r ? 2 : 0] = pack_half2(h0, h1);
        qa[t][kb][r ? 3 : 1] = pack_half2(l0, l1);
        csum += mu * ((h0 + l0) + (h1 + l1));
      }
      csum += __shfl_xor_sync(0xffffffffu, csum, 1);
      csum += __shfl_xor_sync(0xffffffffu, csum, 2);
      kconst[t] = make_float2(csum, 1.0f / lam);
    }
  }

  float oc[DT][4], oz[DT][4];
#pragma unroll
  for (int dt = 0; dt < DT; ++dt)
#pragma unroll
    for (int r = 0; r < 4; ++r) oc[dt][r] = oz[dt][r] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  auto issue = [&](int c) {
    if (c < n_chunks) {
      const int64_t t0 = static_cast<int64_t>(c) * kChunk;
      const int nv = static_cast<int>(p.T - t0 < kChunk ? p.T - t0 : kChunk);
      uint8_t* stg = smem + (c & 1) * STAGE;
      for (int k = threadIdx.x; k < NCHUNK16; k += blockDim.x) {
        const int side = k >= NCHUNK16 / 2;
        int off = (k - side * (NCHUNK16 / 2)) * 16;   // byte offset inside this side
        const uint8_t* base;
        int rec, region;
        if (off < kChunk * CB) { base = side ? p.v_codes : p.k_codes; rec = CB; region = 0; }
        else if (off < kChunk * (CB + SB)) { base = side ? p.v_signs : p.k_signs; rec = SB; region = kChunk * CB; }
        else { base = reinterpret_cast<const uint8_t*>(side ? p.v_norms : p.k_norms); rec = 8; region = kChunk * (CB + SB); }
        const int inreg = off - region;
        const int bytes = max(0, min(16, nv * rec - inreg));
        const uint8_t* src = base + (seq + t0) * rec + inreg;
        cp_async16(stg + side * HALF + off, bytes ? src : base, bytes);
      }
    }
    cp_async_commit();
  };

  issue(0);
#pragma unroll 1
  for (int c = 0; c < n_chunks; ++c) {
    issue(c + 1);
    cp_async_wait<1>();
    __syncthreads();
    const uint8_t* stg = smem + (c & 1) * STAGE;
    const uint8_t* kcd = stg;
    const uint8_t* ksg = stg + kChunk * CB;
    const float2* knm = reinterpret_cast<const float2*>(stg + kChunk * (CB + SB));
    const uint8_t* vcd = stg + HALF;
    const uint8_t* vsg = vcd + kChunk * CB;
    const float2* vnm = reinterpret_cast<const float2*>(vcd + kChunk * (CB + SB));
    const int64_t t0 = static_cast<int64_t>(c) * kChunk;
    const int nv = static_cast<int>(p.T - t0 < kChunk ? p.T - t0 : kChunk);
    const int n_tiles = (nv + 15) / 16;

#pragma unroll 1
    for (int tt = 0; tt < n_tiles; ++tt) {
      const int kbase = tt * 16;
      // ---------------- scores of query gid vs keys kbase + 8 nt + 2 tig + e ----
      float code[2][2], zsc[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) code[nt][0] = code[nt][1] = zsc[nt][0] = zsc[nt][1] = 0.f;
      uint32_t wk[2][P + 1];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int key = kbase + 8 * nt + gid;
        uint32_t raw[BITS];
#pragma unroll
        for (int k = 0; k < BITS; ++k) {
          if constexpr (D == 128) {
            raw[k] = reinterpret_cast<const uint32_t*>(kcd + key * CB + k * (D / 8))[tig];
          } else {
            const uint32_t hw = reinterpret_cast<const uint16_t*>(kcd + key * CB + k * (D / 8))[tig];
            raw[k] = __byte_perm(hw, 0u, 0x4140);   // bytes (b0, 0, b1, 0): bit j+8 -> j+16
          }
        }
        uint32_t pl[P];
        Planes<BITS>::make(raw, pl);
#pragma unroll
        for (int q = 0; q < P; ++q) wk[nt][q] = pl[q];
        if constexpr (D == 128) {
          wk[nt][P] = reinterpret_cast<const uint32_t*>(ksg + key * SB)[tig];
        } else {
          const uint32_t hw = reinterpret_cast<const uint16_t*>(ksg + key * SB)[tig];
          wk[nt][P] = __byte_perm(hw, 0u, 0x4140);
        }
      }
#pragma unroll
      for (int pl = 0; pl <= P; ++pl) {
        const int type = pl < P ? 0 : 1;
        float cc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) cc[nt][0] = cc[nt][1] = cc[nt][2] = cc[nt][3] = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const uint32_t w = wk[nt][pl], ws = w << 8;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            mma_f16(cc[nt], qa[type][kb], bit_pair_h(w, ws, 2 * kb, p.one_h), bit_pair_h(w, ws, 2 * kb + 1, p.one_h));
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float sv = (cc[nt][e] + cc[nt][2 + e] - kconst[type].x) * kconst[type].y;
            if (pl < P) code[nt][e] = fmaf(p.walsh_k[pl < P ? pl : 0], sv, code[nt][e]);
            else zsc[nt][e] = sv;
          }
      }
      float logit[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = kbase + 8 * nt + 2 * tig + e;
          const float2 kn = knm[key];
          const float s = fmaf(kn.x, code[nt][e], kn.y * p.qjl_k * zsc[nt][e]) * p.score_scale;
          logit[nt][e] = key < nv ? s : -INFINITY;
        }
      // ---------------- online softmax for query gid -------------------------
      float mx = fmaxf(fmaxf(logit[0][0], logit[0][1]), fmaxf(logit[1][0], logit[1][1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      if (mx > m_run + kLazyRescale) {
        const float alpha = exp2f(m_run - mx);
        l_run *= alpha;
#pragma unroll
        for (int dt = 0; dt < DT; ++dt)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            oc[dt][r] *= alpha;
            oz[dt][r] *= alpha;
          }
        m_run = mx;
      }
      float pr[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          pr[nt][e] = logit[nt][e] == -INFINITY ? 0.f : exp2f(logit[nt][e] - m_run);
          l_run += pr[nt][e];
        }
      // ---------------- values: A = p * weight pieces, B = +-1 planes ----------
      float wv[2][2], wr[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float2 vn = vnm[kbase + 8 * nt + 2 * tig + e];
          wv[nt][e] = pr[nt][e] * vn.x;
          wr[nt][e] = pr[nt][e] * vn.y;
        }
      // value words: keys kbase + 2 tig (+1), kbase + 8 + 2 tig (+1); this
      // lane's dims are gid*D/8 .. gid*D/8 + D/8 - 1 (byte / half-word gid)
      uint32_t x01[P + 1], x23[P + 1];
      {
        const int k0 = kbase + 2 * tig, k2 = kbase + 8 + 2 * tig;
        uint32_t r01[BITS], r23[BITS];
#pragma unroll
        for (int k = 0; k < BITS; ++k) {
          if constexpr (D == 128) {
            const uint32_t* a = reinterpret_cast<const uint32_t*>(vcd + k * (D / 8));
            const int sel = (gid & 1) ? 0x7632 : 0x5410;
            r01[k] = __byte_perm(a[(k0 * CB) / 4 + (gid >> 1)], a[((k0 + 1) * CB) / 4 + (gid >> 1)], sel);
            r23[k] = __byte_perm(a[(k2 * CB) / 4 + (gid >> 1)], a[((k2 + 1) * CB) / 4 + (gid >> 1)], sel);
          } else {
            const uint8_t* a = vcd + k * (D / 8) + gid;
            r01[k] = static_cast<uint32_t>(a[k0 * CB]) | (static_cast<uint32_t>(a[(k0 + 1) * CB]) << 16);
            r23[k] = static_cast<uint32_t>(a[k2 * CB]) | (static_cast<uint32_t>(a[(k2 + 1) * CB]) << 16);
          }
        }
        uint32_t pl01[P], pl23[P];
        Planes<BITS>::make(r01, pl01);
        Planes<BITS>::make(r23, pl23);
#pragma unroll
        for (int q = 0; q < P; ++q) {
          x01[q] = pl01[q];
          x23[q] = pl23[q];
        }
        if constexpr (D == 128) {
          const uint32_t* a = reinterpret_cast<const uint32_t*>(vsg);
          const int sel = (gid & 1) ? 0x7632 : 0x5410;
          x01[P] = __byte_perm(a[(k0 * SB) / 4 + (gid >> 1)], a[((k0 + 1) * SB) / 4 + (gid >> 1)], sel);
          x23[P] = __byte_perm(a[(k2 * SB) / 4 + (gid >> 1)], a[((k2 + 1) * SB) / 4 + (gid >> 1)], sel);
        } else {
          const uint8_t* a = vsg + gid;
          x01[P] = static_cast<uint32_t>(a[k0 * SB]) | (static_cast<uint32_t>(a[(k0 + 1) * SB]) << 16);
          x23[P] = static_cast<uint32_t>(a[k2 * SB]) | (static_cast<uint32_t>(a[(k2 + 1) * SB]) << 16);
        }
      }
#pragma unroll
      for (int pl = 0; pl <= P; ++pl) {
        // A: rows gid (hi piece) / gid + 8 (lo piece), keys (2tig, 2tig+1), (8+2tig, 8+2tig+1)
        uint32_t a[4];
        {
          float w[2][2];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) w[nt][e] = pl < P ? p.walsh_v[pl < P ? pl : 0] * wv[nt][e] : wr[nt][e];
          // hi = w rounded to bf16, lo = (w - hi) rounded: |w - hi - lo| <= 2^-17 |w|
          uint32_t hi[2][2], lo[2][2];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              hi[nt][e] = bf16_round_bits(w[nt][e]);
              lo[nt][e] = bf16_round_bits(w[nt][e] - __uint_as_float(hi[nt][e]));
            }
          a[0] = __byte_perm(hi[0][0], hi[0][1], 0x7632);
          a[1] = __byte_perm(lo[0][0], lo[0][1], 0x7632);
          a[2] = __byte_perm(hi[1][0], hi[1][1], 0x7632);
          a[3] = __byte_perm(lo[1][0], lo[1][1], 0x7632);
        }
#pragma unroll
        for (int dt = 0; dt < DT; ++dt) {
          if (pl < P) mma_bf16(oc[dt], a, pm1_pair(x01[pl], dt), pm1_pair(x23[pl], dt));
          else mma_bf16(oz[dt], a, pm1_pair(x01[P], dt), pm1_pair(x23[P], dt));
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- epilogue: per query, y = (O_code + qjl S^T O_z) / l, out = Pi^T y ----
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  __syncthreads();
  float* wbuf = reinterpret_cast<float*>(smem) + warp * kQPerWarp * 2 * D;   // [8][2][D]
  const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
#pragma unroll
  for (int dt = 0; dt < DT; ++dt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int dim = (2 * tig + e) * (D / 8) + dt;
      wbuf[(gid * 2 + 0) * D + dim] = (oc[dt][e] + oc[dt][2 + e]) * inv_l;
      wbuf[(gid * 2 + 1) * D + dim] = (oz[dt][e] + oz[dt][2 + e]) * inv_l;
    }
  __syncwarp();
  constexpr int NJ = D / 32;
  for (int qq = 0; qq < kQPerWarp; ++qq) {
    const int qrow = q0 + qq;
    if (qrow >= p.S) break;
    const float* oc_s = wbuf + (qq * 2 + 0) * D;
    const float* oz_s = wbuf + (qq * 2 + 1) * D;
    float y[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int i = lane + 32 * j;
      float corr = 0.f;
      for (int r = 0; r < D; ++r) corr = fmaf(p.v_s[r * D + i], oz_s[r], corr);   // (S^T O_z)_i
      y[j] = oc_s[i] + p.qjl_v * corr;
    }
#pragma unroll
    for (int s = 0; s < 5; ++s) {
      const bool upper = (lane >> s) & 1;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const float o = __shfl_xor_sync(0xffffffffu, y[j], 1 << s);
        y[j] = upper ? o - y[j] : y[j] + o;
      }
    }
#pragma unroll
    for (int bb = 1; bb < NJ; bb <<= 1)
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        if (j & bb) continue;
        const float a0 = y[j], a1 = y[j | bb];
        y[j] = a0 + a1;
        y[j | bb] = a0 - a1;
      }
    float* o = p.out + (static_cast<int64_t>(bq) * p.S + qrow) * D;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int i = lane + 32 * j;
      o[i] = y[j] * p.v_signs_d[i] * rsqrtf(static_cast<float>(D));
    }
  }
}

// ===========================================================================
// Encoder attention on the tensor core (d = 64, 1- and 2-bit codes).
//
// Every key and value tile serves all 128 queries of a CTA, so its bit planes
// are expanded once per tile into exact +-1 operands in shared memory and the
// two products run as tcgen05 MMAs with fp32 accumulators in tensor memory:
//   scores  D_p[q][key] = sum_slot  A[q][slot] * Kop_p[key][slot]
//           (A = q~ for the code planes, S q~ for the sign plane, as fp16 hi
//           and lo pieces of a per-row power-of-two scaling, both pieces
//           accumulating into the same D; keys as fp16 +-1)
//   values  O_code[q][slot] += sum_(p,key) (P ||v|| w_p)[q][(p,key)] * Vop_p[key][slot]
//           O_z[q][slot]    += sum_key     (P ||r_v||)[q][key]        * Vop_z[key][slot]
//           (bf16 hi and lo pieces of the weights against bf16 +-1 values)
// One shift and one LOP3 put bits b and b + 16 of a plane word into one
// 32-bit operand word, so slot k stands for coordinate
// dim(k) = 32 (k / 32) + (k / 2) % 16 + 16 (k % 2) in the queries, keys,
// values and output columns alike; the epilogue undoes it.  The key operand
// (K-major, a row per key) and the value operand (MN-major, a row per key)
// share one physical layout.
//
// A CTA owns 128 queries of one head.  16 worker warps, four threads per
// query row (tensor-memory lane): warp w reads lane quarter w % 4 and keys
// 8 (w / 4) .. + 7 of each 32-key tile; the quarters exchange their tile
// maxima through shared memory.  A 17th warp only issues the MMAs: it waits
// on mbarriers the workers arrive on (operands expanded, probabilities
// written) and commits the products to mbarriers the workers wait on, so the
// issue of the MMAs never holds up a worker barrier.  The loop is
// software-pipelined over tiles: while the workers run the softmax of tile
// i, the tensor core computes the scores of tile i + 1 (two score buffers in
// tensor memory, two key and value operand buffers in shared memory), and
// the packed records of tile i + 2 are in flight (cp.async); the key and
// value operands rotate through three buffers, so the value products of
// tile i - 1 may still run while tile i + 1 is expanded, and the workers wait
// for them only before they rewrite the probability operands.  Every wait is
// bounded; the rows of a CTA whose wait ran out are written as NaN (after a
// failed wait the MMA warp stops issuing but still commits, so no wait of
// the workers is left without its arrival).
// ===========================================================================
constexpr int kTcQ = 128;               // queries per CTA
constexpr int kTcKeys = 32;             // keys per tile
constexpr int kTcWorkers = 512;         // 16 worker warps, four threads per query row
constexpr int kTcThreads = kTcWorkers + 32;   // and the MMA warp
constexpr int kTcWait = 1 << 17;        // polls of about 9 us each
constexpr int kTcOpQ = kTcQ * 128;      // one [128 x 64] 16-bit operand: 16 KB
constexpr int kTcOpK = kTcKeys * 128;   // one [32 x 64] 16-bit operand: 4 KB
constexpr int kTcEpiB = 64 * 128;      // one [64 x 64] bf16 operand of the output transform: 8 KB
constexpr uint32_t kTcColO = 256;       // tensor-memory columns: scores 0..191 (two buffers), O 256..383

template <int BITS>
__host__ __device__ constexpr int tc_kv_bytes() {
  return 2 * (Planes<BITS>::P + 1) * kTcOpK;   // key and value operands of one tile
}
template <int BITS>
__host__ __device__ constexpr int tc_stage_bytes() {
  return 2 * kTcKeys * (BITS * 8 + 8 + 8);   // K and V sides of one staged tile (d = 64)
}
template <int BITS>
constexpr size_t tc_smem_bytes() {
  return 1024 + 4 * kTcOpQ + 3 * tc_kv_bytes<BITS>() + 3 * kTcOpQ + 2 * tc_stage_bytes<BITS>();
}

// slot k of an operand row -> coordinate
__host__ __device__ constexpr int tc_slot_dim(int k) { return 32 * (k >> 5) + ((k >> 1) & 15) + 16 * (k & 1); }

// byte offset of 16-byte chunk j of row r in a 128-byte swizzled operand
__device__ __forceinline__ uint32_t tc_chunk_off(int r, int j) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

// 8 consecutive slots as fp16 hi and lo pieces: hi = RN(x), lo = RN(x - hi)
__device__ __forceinline__ void tc_split8_h(const float (&x)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __half2 hh = __floats2half2_rn(x[2 * e], x[2 * e + 1]);
    const float2 hf = __half22float2(hh);
    const __half2 ll = __floats2half2_rn(x[2 * e] - hf.x, x[2 * e + 1] - hf.y);
    h[e] = *reinterpret_cast<const uint32_t*>(&hh);
    l[e] = *reinterpret_cast<const uint32_t*>(&ll);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// 8 consecutive slots as bf16 hi and lo pieces: hi = RN(x), lo = RN(x - hi)
__device__ __forceinline__ void tc_split8(const float (&x)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
    h[e] = *reinterpret_cast<uint32_t*>(&hh);
    const float2 d = __ffma2_rn(make_float2(__uint_as_float(h[e] << 16), __uint_as_float(h[e] & 0xFFFF0000u)),
                                make_float2(-1.f, -1.f), make_float2(x[2 * e], x[2 * e + 1]));
    __nv_bfloat162 ll = __floats2bfloat162_rn(d.x, d.y);
    l[e] = *reinterpret_cast<uint32_t*>(&ll);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <int BITS>
__global__ void __launch_bounds__(kTcThreads, 1) encoder_tc_kernel(const __grid_constant__ EncParams p) {
  constexpr int D = 64;
  constexpr int P = Planes<BITS>::P;
  constexpr int CB = BITS * D / 8, SB = D / 8;
  constexpr int HALF = kTcKeys * (CB + SB + 8);
  constexpr int STG = 2 * HALF;
  constexpr int KV = tc_kv_bytes<BITS>();
  static_assert(P <= 2, "code planes of at most 2 bits");
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t mb_s[2], mb_pv, mb_kv, mb_p;   // products done; operands / probabilities ready
  __shared__ uint64_t mb_epi;                        // the output transform's products done
  __shared__ uint32_t tmem_slot;
  __shared__ int s_fail;
  __shared__ float s_inv_lam[2][kTcQ];        // per query row: 1 / range scale of q~ (0) and S q~ (1)
  __shared__ float s_mx[4][kTcQ];             // per key quarter, query row: tile maximum of the logits
  __shared__ __align__(16) float2 s_kf[2][kTcKeys];   // per tile buffer, key: (||k||, ||r_k|| qjl_k) x score scale
  __shared__ __align__(16) float s_vf[3][2][kTcKeys];  // per factor, tile buffer, key: ||v|| w_0, ||v|| w_1, ||r_v||
  uint8_t* base = raw + ((1024 - (tqtc::smem_u32(raw) & 1023)) & 1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kq = warp >> 2;                   // key quarter of this thread in the softmax
  const int row = 32 * (warp & 3) + lane;     // query row = tensor-memory lane
  uint8_t* aq_hi = base;                      // q~ pieces (rows = queries)
  uint8_t* aq_lo = base + kTcOpQ;
  uint8_t* as_hi = base + 2 * kTcOpQ;         // S q~ pieces
  uint8_t* as_lo = base + 3 * kTcOpQ;
  uint8_t* kvb = base + 4 * kTcOpQ;           // three buffers: key operand planes, then value operand rows
  uint8_t* ac_hi = kvb + 3 * KV;              // rows = queries, slots (pl, key)
  uint8_t* ac_lo = ac_hi + kTcOpQ;
  uint8_t* az = ac_lo + kTcOpQ;               // slots key: hi piece, 32 + key: lo piece
  uint8_t* stg = az + kTcOpQ;                 // two staged tiles

  const int bq = blockIdx.y;
  const int b = bq / p.Hq, h = bq % p.Hq;
  const int bh = b * (p.Hq / p.G) + h / p.G;
  const int q0 = blockIdx.x * kTcQ;
  const int64_t seq = static_cast<int64_t>(bh) * p.cache_stride;
  const int n_tiles = static_cast<int>((p.T + kTcKeys - 1) / kTcKeys);

  const bool mma_warp = warp == kTcWorkers / 32;
  if (tid == 0) {
    tqtc::mbar_init(&mb_s[0], 1);
    tqtc::mbar_init(&mb_s[1], 1);
    tqtc::mbar_init(&mb_pv, 1);
    tqtc::mbar_init(&mb_kv, kTcWorkers);
    tqtc::mbar_init(&mb_p, kTcWorkers);
    tqtc::mbar_init(&mb_epi, 1);
    s_fail = 0;
  }
  if (warp == 0) tqtc::tmem_alloc(&tmem_slot, 512);

  auto issue = [&](int t) {   // stage tile t into buffer t & 1
    if (t < n_tiles) {
      const int64_t t0 = static_cast<int64_t>(t) * kTcKeys;
      const int nv = static_cast<int>(p.T - t0 < kTcKeys ? p.T - t0 : kTcKeys);
      uint8_t* dst = stg + (t & 1) * STG;
      for (int c = tid; c < STG / 16; c += kTcWorkers) {
        const int side = c >= STG / 32;
        const int off = (c - side * (STG / 32)) * 16;   // byte offset inside this side
        const uint8_t* src_base;
        int rec, region;
        if (off < kTcKeys * CB) {
          src_base = side ? p.v_codes : p.k_codes;
          rec = CB;
          region = 0;
        } else if (off < kTcKeys * (CB + SB)) {
          src_base = side ? p.v_signs : p.k_signs;
          rec = SB;
          region = kTcKeys * CB;
        } else {
          src_base = reinterpret_cast<const uint8_t*>(side ? p.v_norms : p.k_norms);
          rec = 8;
          region = kTcKeys * (CB + SB);
        }
        const int inreg = off - region;
        const int bytes = max(0, min(16, nv * rec - inreg));
        const uint8_t* src = src_base + (seq + t0) * rec + inreg;
        cp_async16(dst + side * HALF + off, bytes ? src : src_base, bytes);
      }
    }
    cp_async_commit();
  };
  if (!mma_warp) {
    issue(0);
    issue(1);
  }

  // ---- query operands: thread (row, kq) writes slots 16 kq .. 16 kq + 15 of
  // q~ (kq < 2) or S q~ (kq >= 2) as fp16 hi and lo pieces of x * lam, lam a
  // power of two bringing the row's max |x| into [2^13, 2^14) (about 22
  // significant bits); the key operand is fp16 too
  if (!mma_warp) {
    const int q = q0 + row, type = kq >> 1, half = kq & 1;
    float v[32];   // coordinates 32 half .. 32 half + 31
    float mx = 0.f;
    if (q < p.S) {
      const float4* src =
          reinterpret_cast<const float4*>(p.qprep + ((static_cast<int64_t>(bq) * p.S + q) * 2 + type) * D);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 f = src[8 * half + i];
        v[4 * i] = f.x;
        v[4 * i + 1] = f.y;
        v[4 * i + 2] = f.z;
        v[4 * i + 3] = f.w;
        const float4 o = src[8 * (1 - half) + i];
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(v[i]));
    const float lam = fp16_range_scale(mx);
    if (half == 0) s_inv_lam[type][row] = 1.f / lam;
    uint8_t* dhi = type ? as_hi : aq_hi;
    uint8_t* dlo = type ? as_lo : aq_lo;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float x[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = v[tc_slot_dim(8 * j + e)] * lam;   // slot 32 half + 8 j + e
      uint4 hi, lo;
      tc_split8_h(x, hi, lo);
      *reinterpret_cast<uint4*>(dhi + tc_chunk_off(row, 4 * half + j)) = hi;
      *reinterpret_cast<uint4*>(dlo + tc_chunk_off(row, 4 * half + j)) = lo;
    }
  }

  // ---- expansion of tile t (staged in buffer t & 1) into operand buffer t % 3:
  // thread -> key tid / 16, side (tid / 8) % 2, chunk tid % 8 of every plane
  const int xkey = tid >> 4, xside = (tid >> 3) & 1, xj = tid & 7;
  auto expand = [&](int t) {
    const uint8_t* sd = stg + (t & 1) * STG + xside * HALF;
    uint32_t rw[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) rw[k] = reinterpret_cast<const uint32_t*>(sd + xkey * CB + k * (D / 8))[xj >> 2];
    uint32_t pw[P + 1];
    {
      uint32_t pl[P];
      Planes<BITS>::make(rw, pl);
#pragma unroll
      for (int q = 0; q < P; ++q) pw[q] = pl[q];
    }
    pw[P] = reinterpret_cast<const uint32_t*>(sd + kTcKeys * CB + xkey * SB)[xj >> 2];
    const uint32_t one = xside ? 0x3F803F80u : 0x3C003C00u;   // +1 in both halves: bf16 values, fp16 keys
    uint8_t* dst = kvb + (t % 3) * KV + xside * (P + 1) * kTcOpK;
#pragma unroll
    for (int pl = 0; pl <= P; ++pl) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t s = pw[pl] << (15 - (4 * (xj & 3) + e));
        w4[e] = (~s & 0x80008000u) | one;
      }
      *reinterpret_cast<uint4*>(dst + pl * kTcOpK + tc_chunk_off(xkey, xj)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    if (tid < kTcKeys) {
      const uint8_t* s0 = stg + (t & 1) * STG;
      const float2 kn = reinterpret_cast<const float2*>(s0 + kTcKeys * (CB + SB))[tid];
      const float2 vn = reinterpret_cast<const float2*>(s0 + HALF + kTcKeys * (CB + SB))[tid];
      s_kf[t & 1][tid] = make_float2(kn.x * p.score_scale, kn.y * p.qjl_k * p.score_scale);
      s_vf[0][t & 1][tid] = vn.x * p.walsh_v[0];
      s_vf[1][t & 1][tid] = vn.x * p.walsh_v[1];
      s_vf[2][t & 1][tid] = vn.y;
    }
  };

  tqtc::fence_smem_to_async();
  tqtc::fence_before_sync();
  __syncthreads();
  tqtc::fence_after_sync();
  const uint32_t tmem = tmem_slot;
  const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);   // this warp's lanes
  // descriptors (the leader issues): a k step adds 32 bytes along K (2 units),
  // an MN-major k step 16 rows (2048 bytes, 128 units)
  const uint64_t dq_hi = tqtc::sw128_desc(tqtc::smem_u32(aq_hi)), dq_lo = tqtc::sw128_desc(tqtc::smem_u32(aq_lo));
  const uint64_t ds_hi = tqtc::sw128_desc(tqtc::smem_u32(as_hi)), ds_lo = tqtc::sw128_desc(tqtc::smem_u32(as_lo));
  const uint64_t dkv = tqtc::sw128_desc(tqtc::smem_u32(kvb)), dkv_mn = tqtc::sw128_desc_mn(tqtc::smem_u32(kvb));
  const uint64_t dc_hi = tqtc::sw128_desc(tqtc::smem_u32(ac_hi)), dc_lo = tqtc::sw128_desc(tqtc::smem_u32(ac_lo));
  const uint64_t dz = tqtc::sw128_desc(tqtc::smem_u32(az));
  auto issue_scores = [&](int t) {   // D[t & 1] = q pieces x key operand of tile t
    constexpr uint32_t idesc = tqtc::idesc_f16_f32(kTcQ, kTcKeys);
    const uint32_t dcol = tmem + 96 * (t & 1);
    const uint64_t kb = dkv + static_cast<uint64_t>(((t % 3) * KV) >> 4);
#pragma unroll
    for (int pl = 0; pl <= P; ++pl) {
      const uint64_t a_hi = pl < P ? dq_hi : ds_hi, a_lo = pl < P ? dq_lo : ds_lo;
      const uint64_t bk = kb + static_cast<uint64_t>((pl * kTcOpK) >> 4);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) tqtc::mma_bf16_ss(dcol + 32 * pl, a_hi + 2 * ks, bk + 2 * ks, idesc, ks > 0);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) tqtc::mma_bf16_ss(dcol + 32 * pl, a_lo + 2 * ks, bk + 2 * ks, idesc, true);
    }
  };
  auto issue_values = [&](int t) {   // O += probability operands x value operand of tile t
    constexpr uint32_t idesc = tqtc::idesc_bf16_f32(kTcQ, D) | tqtc::kIdescBMajorMN;
    const bool acc = t > 0;
    const uint64_t vc = dkv_mn + static_cast<uint64_t>(((t % 3) * KV + (P + 1) * kTcOpK) >> 4);
    const uint64_t vz = vc + static_cast<uint64_t>((P * kTcOpK) >> 4);
    const uint32_t ocode = tmem + kTcColO, oz = tmem + kTcColO + 64;
#pragma unroll
    for (int ks = 0; ks < 2 * P; ++ks) tqtc::mma_bf16_ss(ocode, dc_hi + 2 * ks, vc + 128 * ks, idesc, acc || ks > 0);
#pragma unroll
    for (int ks = 0; ks < 2 * P; ++ks) tqtc::mma_bf16_ss(ocode, dc_lo + 2 * ks, vc + 128 * ks, idesc, true);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) tqtc::mma_bf16_ss(oz, dz + 2 * ks, vz + 128 * (ks & 1), idesc, acc || ks > 0);
  };

  if (mma_warp) {
    // ---- MMA issue: scores of tile t + 1 as soon as its operands are
    // expanded, values of tile t as soon as its probabilities are written
    if (lane == 0) {
      bool mok = true;
      auto ready = [&](uint64_t* mb, int t) {
        mok = mok && s_fail == 0 && tqtc::mbar_wait(mb, t & 1, kTcWait);
        if (!mok) s_fail = 1;
        tqtc::fence_after_sync();
        return mok;
      };
      if (n_tiles > 0) {
        if (ready(&mb_kv, 0)) issue_scores(0);
        tqtc::mma_commit(&mb_s[0]);
      }
      for (int t = 0; t < n_tiles; ++t) {
        if (t + 1 < n_tiles) {
          if (ready(&mb_kv, t + 1)) issue_scores(t + 1);
          tqtc::mma_commit(&mb_s[(t + 1) & 1]);
        }
        if (ready(&mb_p, t)) issue_values(t);
        tqtc::mma_commit(&mb_pv);
      }
    }
    __syncwarp();
  } else {

  auto work_sync = [&]() { asm volatile("bar.sync 1, %0;\n" ::"n"(kTcWorkers) : "memory"); };
  // one lane polls an mbarrier for the warp (all lanes polling the same word
  // serialise in shared memory); the shuffle orders the other lanes after it
  auto warp_wait = [&](uint64_t* mb, uint32_t parity) {
    int done = 0;
    if (lane == 0) done = tqtc::mbar_wait(mb, parity, kTcWait) ? 1 : 0;
    return __shfl_sync(0xffffffffu, done, 0) != 0;
  };
  // prologue: tile 0 expanded
  bool ok = true;
  if (n_tiles > 0) {
    cp_async_wait<1>();
    work_sync();
    expand(0);
    tqtc::fence_smem_to_async();
    tqtc::fence_before_sync();
    tqtc::mbar_arrive(&mb_kv);
  }
  float m_run = -INFINITY, l_run = 0.f;
  uint32_t ph_s0 = 0, ph_s1 = 0, ph_pv = 0;
  bool pv_pending = false;   // value products issued and not yet waited for (CTA-uniform)
#pragma unroll 1
  for (int it = 0; it < n_tiles; ++it) {
    const bool has_next = it + 1 < n_tiles;
    cp_async_wait<0>();
    work_sync();   // tile it + 1 is staged; buffer it & 1 of the staging is free
    issue(it + 2);
    // scores of tile it (issued one iteration earlier; waiting for them here
    // also means the MMA warp has taken this tile's operand signal, so the
    // next signal cannot complete a phase it has not yet waited for)
    {
      uint32_t& ph = (it & 1) ? ph_s1 : ph_s0;
      ok = warp_wait(&mb_s[it & 1], ph) && ok;
      ph ^= 1;
    }
    tqtc::fence_after_sync();
    if (has_next) {
      expand(it + 1);
      tqtc::fence_smem_to_async();
      tqtc::fence_before_sync();
      tqtc::mbar_arrive(&mb_kv);
    }
    const int64_t t0 = static_cast<int64_t>(it) * kTcKeys;
    const int nv = static_cast<int>(p.T - t0 < kTcKeys ? p.T - t0 : kTcKeys);

    // ---- logits of query `row` against keys 8 kq .. 8 kq + 7 of tile it
    float lg[8];
    {
      float d0[8], d1[8], dzv[8];
      const uint32_t dcol = tl + 96 * (it & 1) + 8 * kq;
      tqtc::tmem_ld8x3(dcol, dcol + 32 * (P - 1), dcol + 32 * P, d0, d1, dzv);
      const float iq = s_inv_lam[0][row], iz = s_inv_lam[1][row];
      const float wq0 = p.walsh_k[0] * iq, wq1 = p.walsh_k[1] * iq;
      const float2 wq0_2 = make_float2(wq0, wq0), wq1_2 = make_float2(wq1, wq1), iz_2 = make_float2(iz, iz);
      // two keys per fp32x2 instruction (the same roundings as one key at a time)
#pragma unroll
      for (int k = 0; k < 8; k += 2) {
        const float4 kf = *reinterpret_cast<const float4*>(&s_kf[it & 1][8 * kq + k]);   // keys k, k + 1
        float2 c = __fmul2_rn(wq0_2, make_float2(d0[k], d0[k + 1]));
        if constexpr (P == 2) c = __ffma2_rn(wq1_2, make_float2(d1[k], d1[k + 1]), c);
        const float2 zt = __fmul2_rn(__fmul2_rn(make_float2(kf.y, kf.w), iz_2), make_float2(dzv[k], dzv[k + 1]));
        const float2 l2 = __ffma2_rn(make_float2(kf.x, kf.z), c, zt);
        lg[k] = l2.x;
        lg[k + 1] = l2.y;
      }
    }
    if (nv < kTcKeys) {
#pragma unroll
      for (int k = 0; k < 8; ++k) lg[k] = 8 * kq + k < nv ? lg[k] : -INFINITY;
    }
    float mloc = lg[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) mloc = fmaxf(mloc, lg[k]);
    s_mx[kq][row] = mloc;
    work_sync();
    // the previous value products read the probability operands rewritten
    // below and accumulate the O rescaled below (the MMA warp commits even
    // after a failure, so this wait always ends)
    if (pv_pending) {
      ok = warp_wait(&mb_pv, ph_pv) && ok;
      ph_pv ^= 1;
      pv_pending = false;
    }
    tqtc::fence_after_sync();
    const bool failed = __any_sync(0xffffffffu, !ok || s_fail != 0);   // warp-uniform (tensor-memory access below)
    const float mx = fmaxf(fmaxf(s_mx[0][row], s_mx[1][row]), fmaxf(s_mx[2][row], s_mx[3][row]));
    const bool need = mx > m_run + kLazyRescale;   // the same in the four threads of the row
    if (__any_sync(0xffffffffu, need)) {
      const float alpha = need ? exp2_approx(m_run - mx) : 1.f;
      if (it > 0 && !failed) {
        // this thread's quarter of O (columns 32 kq ..), rescaled in tensor
        // memory (the previous value products are complete)
        float o[32];
        const uint32_t a = tl + kTcColO + 32 * kq;
        tqtc::tmem_ld32(a, o);
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] *= alpha;
        tqtc::tmem_st32(a, o);
      }
      l_run *= alpha;
      if (need) m_run = mx;
    }
    // ---- probabilities -> value-product operands (row `row`, keys 8 kq .. + 7)
    {
      float xc[P][8], xz[8], pk[8];
      const float2 nm = make_float2(-m_run, -m_run);
#pragma unroll
      for (int k = 0; k < 8; k += 2) {   // two keys per fp32x2 instruction
        const float2 e = __fadd2_rn(make_float2(lg[k], lg[k + 1]), nm);
        pk[k] = lg[k] == -INFINITY ? 0.f : exp2_approx(e.x);
        pk[k + 1] = lg[k + 1] == -INFINITY ? 0.f : exp2_approx(e.y);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) l_run += pk[k];
#pragma unroll
      for (int f = 0; f < 3; ++f) {
        if (P == 1 && f == 1) continue;
        float* dst = f == 2 ? xz : xc[f < P ? f : 0];
#pragma unroll
        for (int k = 0; k < 8; k += 4) {
          const float4 v = *reinterpret_cast<const float4*>(&s_vf[f][it & 1][8 * kq + k]);
          const float2 a = __fmul2_rn(make_float2(pk[k], pk[k + 1]), make_float2(v.x, v.y));
          const float2 b = __fmul2_rn(make_float2(pk[k + 2], pk[k + 3]), make_float2(v.z, v.w));
          dst[k] = a.x;
          dst[k + 1] = a.y;
          dst[k + 2] = b.x;
          dst[k + 3] = b.y;
        }
      }
      uint4 hi, lo;
#pragma unroll
      for (int pl = 0; pl < P; ++pl) {
        tc_split8(xc[pl], hi, lo);
        *reinterpret_cast<uint4*>(ac_hi + tc_chunk_off(row, 4 * pl + kq)) = hi;
        *reinterpret_cast<uint4*>(ac_lo + tc_chunk_off(row, 4 * pl + kq)) = lo;
      }
      tc_split8(xz, hi, lo);
      *reinterpret_cast<uint4*>(az + tc_chunk_off(row, kq)) = hi;
      *reinterpret_cast<uint4*>(az + tc_chunk_off(row, 4 + kq)) = lo;
    }
    tqtc::fence_smem_to_async();
    tqtc::fence_before_sync();
    tqtc::mbar_arrive(&mb_p);
    pv_pending = true;
    if (!ok) s_fail = 1;
  }
  if (pv_pending) ok = warp_wait(&mb_pv, ph_pv) && ok;
  tqtc::fence_after_sync();
  if (!ok) s_fail = 1;
  cp_async_wait<0>();
  work_sync();   // the operand areas take the epilogue buffers

  // ---- epilogue on the tensor core: out = D H (O_code + qjl S^T O_z) / (8 l)
  // = (O_code B1^T + O_z B2^T) / l with B1 = D H / 8 and B2 = qjl D H S^T / 8
  // in slot order (built with the value handle).  Thread (row, kq) writes O
  // columns 32 kq .. + 31 (O_code for kq < 2, O_z after) as bf16 hi and lo
  // operand rows, one thread issues the 20 MMAs into the first score buffer,
  // and each thread scales and stores its 16 outputs.
  uint8_t* eo = kvb;                            // O_code hi, lo, O_z hi, lo: 4 x [128 x 64] bf16
  uint8_t* eb = kvb + 4 * kTcOpQ;               // B1, B2 hi, B2 lo: 3 x [64 x 64] bf16
  float* lbuf = reinterpret_cast<float*>(eb + 3 * kTcEpiB);   // [4][128]: l of each quarter
  for (int i = tid; i < 3 * kTcEpiB / 16; i += kTcWorkers)
    cp_async16(eb + 16 * i, reinterpret_cast<const uint8_t*>(p.epi) + 16 * i, 16);
  cp_async_commit();
  lbuf[kq * kTcQ + row] = n_tiles > 0 ? l_run : 0.f;
  {
    float o[32];
    tqtc::tmem_ld32(tl + kTcColO + 32 * kq, o);
    uint8_t* ahi = eo + (kq >> 1) * 2 * kTcOpQ;
    uint8_t* alo = ahi + kTcOpQ;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float x[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = n_tiles > 0 ? o[8 * j + e] : 0.f;
      uint4 hi, lo;
      tc_split8(x, hi, lo);
      const int c = 4 * (kq & 1) + j;   // slots 32 (kq % 2) + 8 j .. + 7
      *reinterpret_cast<uint4*>(ahi + tc_chunk_off(row, c)) = hi;
      *reinterpret_cast<uint4*>(alo + tc_chunk_off(row, c)) = lo;
    }
  }
  cp_async_wait<0>();
  tqtc::fence_smem_to_async();
  tqtc::fence_before_sync();
  work_sync();
  if (tid == 0) {
    tqtc::fence_after_sync();
    constexpr uint32_t idesc = tqtc::idesc_bf16_f32(kTcQ, D);
    const uint64_t a0 = tqtc::sw128_desc(tqtc::smem_u32(eo)), b0 = tqtc::sw128_desc(tqtc::smem_u32(eb));
    constexpr uint64_t at = kTcOpQ >> 4, bt = kTcEpiB >> 4;
    // code hi x B1, code lo x B1, z hi x B2 hi, z hi x B2 lo, z lo x B2 hi
    constexpr int pa[5] = {0, 1, 2, 2, 3}, pb[5] = {0, 0, 1, 2, 1};
#pragma unroll
    for (int pr = 0; pr < 5; ++pr)
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tqtc::mma_bf16_ss(tmem, a0 + pa[pr] * at + 2 * ks, b0 + pb[pr] * bt + 2 * ks, idesc, pr > 0 || ks > 0);
    tqtc::mma_commit(&mb_epi);
  }
  const bool eok = warp_wait(&mb_epi, 0);
  tqtc::fence_after_sync();
  const float l = (lbuf[row] + lbuf[kTcQ + row]) + (lbuf[2 * kTcQ + row] + lbuf[3 * kTcQ + row]);
  const float inv_l = l > 0.f ? 1.f / l : 0.f;
  float r0[16], r1[16], r2[16];
  tqtc::tmem_ld16x3(tl + 16 * kq, tl + 16 * kq, tl + 16 * kq, r0, r1, r2);
  const int q = q0 + row;
  if (q < p.S) {
    const bool bad = s_fail != 0 || !eok;
    float4* o = reinterpret_cast<float4*>(p.out + (static_cast<int64_t>(bq) * p.S + q) * D + 16 * kq);
#pragma unroll
    for (int i4 = 0; i4 < 4; ++i4)
      o[i4] = bad ? make_float4(NAN, NAN, NAN, NAN)
                  : make_float4(r0[4 * i4] * inv_l, r0[4 * i4 + 1] * inv_l, r0[4 * i4 + 2] * inv_l,
                                r0[4 * i4 + 3] * inv_l);
  }
  }   // workers
  tqtc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tqtc::tmem_free(tmem, 512);
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

size_t enc_workspace(int B, int Hq, int S, int d) {
  return align256(static_cast<size_t>(B) * Hq * S * 2 * d * sizeof(float));
}

template <int D, int BITS>
int launch_enc(const EncParams& p, int B, cudaStream_t s) {
  constexpr int CB = BITS * D / 8, SB = D / 8;
  const size_t stage = 2 * static_cast<size_t>(kChunk) * (CB + SB + 8);
  const size_t epi = static_cast<size_t>(kWarps) * kQPerWarp * 2 * D * sizeof(float);
  const size_t smem = 2 * stage > epi ? 2 * stage : epi;
  auto kern = encoder_attention_kernel<D, BITS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return TQ_ECUDA;
  dim3 grid((p.S + kWarps * kQPerWarp - 1) / (kWarps * kQPerWarp), B * p.Hq);
  kern<<<grid, kWarps * 32, smem, s>>>(p);
  return tq::launch_status();
}

template <int BITS>
int launch_enc_tc(const EncParams& p, int B, cudaStream_t s) {
  constexpr size_t smem = tc_smem_bytes<BITS>();
  static_assert(smem <= 227 * 1024, "shared memory of the tensor-core encoder kernel");
  auto kern = encoder_tc_kernel<BITS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return TQ_ECUDA;
  dim3 grid((p.S + kTcQ - 1) / kTcQ, B * p.Hq);
  kern<<<grid, kTcThreads, smem, s>>>(p);
  return tq::launch_status();
}

template <int D>
int dispatch_bits(int bits, const EncParams& p, int B, cudaStream_t s) {
  switch (bits) {
    case 1: return launch_enc<D, 1>(p, B, s);
    case 2: return launch_enc<D, 2>(p, B, s);
    case 3: return launch_enc<D, 3>(p, B, s);
  }
  return TQ_EUNSUPPORTED;
}

}  // namespace

extern "C" size_t tq_encoder_workspace_size(const tq_rotation* hk, int B, int Hq, int S) {
  if (!hk || B < 1 || Hq < 1 || S < 1) return 0;
  return enc_workspace(B, Hq, S, hk->d);
}

extern "C" int tq_encoder_attention(const tq_rotation* hk, const tq_rotation* hv, const void* q, int q_dtype,
                                    int64_t q_pos_offset, const uint8_t* k_codes, const uint8_t* k_signs,
                                    const float* k_norms, const uint8_t* v_codes, const uint8_t* v_signs,
                                    const float* v_norms, int64_t cache_stride, int B, int Hq, int Hkv, int S,
                                    int64_t T, float scale, float* out, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  if (!hk || !hv || !q || !out) return TQ_EINVAL;
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || S < 1 || T < 0 || !std::isfinite(scale)) return TQ_EINVAL;
  if (hk->d != hv->d || hk->m != hv->m || hk->bits != hv->bits) return TQ_EINVAL;
  if (hk->kind != TQ_ROT_HADAMARD || hv->kind != TQ_ROT_HADAMARD) return TQ_EUNSUPPORTED;
  const int d = hk->d;
  if (d != 64 && d != 128) return TQ_EUNSUPPORTED;
  if (T > 0) {
    if (!k_codes || !k_signs || !k_norms || !v_codes || !v_signs || !v_norms) return TQ_EINVAL;
    if (cache_stride < T || (cache_stride & 1)) return TQ_EINVAL;
    const void* ptrs[6] = {k_codes, k_signs, k_norms, v_codes, v_signs, v_norms};
    for (const void* ptr : ptrs)
      if (!tq::aligned16(ptr)) return TQ_EINVAL;
  }
  if (hk->rope_base > 0.0) {
    if (q_pos_offset < 0 || q_pos_offset + S > hk->rope_max_pos) return TQ_EINVAL;
  }
  const size_t need = enc_workspace(B, Hq, S, d);
  if (!workspace || workspace_bytes < need) return TQ_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TQ_EINVAL;
  if (!tq::on_handle_device(hk) || !tq::on_handle_device(hv)) return TQ_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* qp = static_cast<float*>(workspace);
  const int64_t nq = static_cast<int64_t>(B) * Hq * S;
  const int qblocks = static_cast<int>((nq + 7) / 8);
  const int rope = hk->rope_base > 0.0 ? 1 : 0;
  if (d == 64) {
    if (q_dtype == TQ_F32)
      encoder_qprep_kernel<64, float><<<qblocks, 256, 0, s>>>(static_cast<const float*>(q), nq, S, q_pos_offset,
                                                               hk->d_signs, hk->d_st, hk->d_rope_hi, hk->d_rope_lo,
                                                               hk->rope_max_pos, rope, qp);
    else
      encoder_qprep_kernel<64, __nv_bfloat16><<<qblocks, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(q), nq, S, q_pos_offset, hk->d_signs, hk->d_st, hk->d_rope_hi,
          hk->d_rope_lo, hk->rope_max_pos, rope, qp);
  } else {
    if (q_dtype == TQ_F32)
      encoder_qprep_kernel<128, float><<<qblocks, 256, 0, s>>>(static_cast<const float*>(q), nq, S, q_pos_offset,
                                                                hk->d_signs, hk->d_st, hk->d_rope_hi, hk->d_rope_lo,
                                                                hk->rope_max_pos, rope, qp);
    else
      encoder_qprep_kernel<128, __nv_bfloat16><<<qblocks, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(q), nq, S, q_pos_offset, hk->d_signs, hk->d_st, hk->d_rope_hi,
          hk->d_rope_lo, hk->rope_max_pos, rope, qp);
  }
  int st = tq::launch_status();
  if (st != TQ_OK) return st;
  EncParams p{};
  p.qprep = qp;
  p.k_codes = k_codes;
  p.k_signs = k_signs;
  p.k_norms = reinterpret_cast<const float2*>(k_norms);
  p.v_codes = v_codes;
  p.v_signs = v_signs;
  p.v_norms = reinterpret_cast<const float2*>(v_norms);
  p.cache_stride = cache_stride;
  p.T = T;
  p.S = S;
  p.Hq = Hq;
  p.G = Hq / Hkv;
  p.score_scale = scale * 1.4426950408889634f;
  p.qjl_k = static_cast<float>(hk->res_const);
  p.one_h = kOneH2;
  p.one_b = kOneB2;
  p.qjl_v = static_cast<float>(hv->res_const);
  for (int i = 0; i < 4; ++i) {
    p.walsh_k[i] = static_cast<float>(hk->walsh[i]);
    p.walsh_v[i] = static_cast<float>(hv->walsh[i]);
  }
  p.v_s = hv->d_s;
  p.v_signs_d = hv->d_signs;
  p.out = out;
  // d = 64 with 1- or 2-bit codes and m = d: tensor-core kernel; otherwise the mma.sync kernel
  p.epi = hv->d_enc_epi;
  if (d == 64 && hk->m == 64 && hk->bits <= 2 && hv->d_enc_epi && tq::aligned16(out))
    return hk->bits == 1 ? launch_enc_tc<1>(p, B, s) : launch_enc_tc<2>(p, B, s);
  return d == 64 ? dispatch_bits<64>(hk->bits, p, B, s) : dispatch_bits<128>(hk->bits, p, B, s);
}
