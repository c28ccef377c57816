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
// Walsh-Hadamard rotation, S q~) and the attention kernel.  The attention
// kernel is flash-attention shaped on mma.sync m16n8k16 (bf16 in, fp32
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
  p.qjl_k = static_cast<float>(kQjlConst / hk->m);
  p.one_h = kOneH2;
  p.one_b = kOneB2;
  p.qjl_v = static_cast<float>(kQjlConst / hv->m);
  for (int i = 0; i < 4; ++i) {
    p.walsh_k[i] = static_cast<float>(hk->walsh[i]);
    p.walsh_v[i] = static_cast<float>(hv->walsh[i]);
  }
  p.v_s = hv->d_s;
  p.v_signs_d = hv->d_signs;
  p.out = out;
  return d == 64 ? dispatch_bits<64>(hk->bits, p, B, s) : dispatch_bits<128>(hk->bits, p, B, s);
}
