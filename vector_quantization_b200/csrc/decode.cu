// Decode attention scored straight from the packed K/V cache.
//
// [TurboESM] §2.E: dequantization, residual correction, inverse rotation
// Pi^T and an online softmax fused into one pass over the cache, with no
// dequantized intermediate in memory.  [TurboQuant] "QJL": the score of a
// key is <q~, ||k|| c[idx]> + ||r|| sqrt(pi/2)/m <S q~, sign(S r)>, q~ = Pi q.
//
// Three launches per call:
//  1. qprep   - per query head: RoPE, q~ = Pi q (fast Walsh-Hadamard),
//               s = S q~; both written as bf16 hi/lo pairs directly in the
//               register order of the main kernel's MMA B operand.
//  2. split   - per (sequence, token chunk): streams the packed records
//               through shared memory (cp.async, 4-stage ring per warp),
//               scores 16 tokens at a time and accumulates the values.  The
//               loop is software-pipelined: the key-side products of tile i
//               and the value-side products of tile i-1 sit in one loop body,
//               so the two tensor-core streams overlap; the online-softmax
//               rescale runs after both, which keeps it exact.
//  3. merge   - per query head: log-sum-exp merge of the chunk partials, the
//               QJL value correction S^T acc_s, and Pi^T.
//
// The contraction trick.  A b-bit code is rewritten in Walsh form,
//   c[idx] = sum_p w_p s_p(idx),  s_p a product of the code's bits as +-1,
// (b = 2: s_1, s_0; b = 3: s_2, s_1, s_0, s_0 s_1 s_2), and the QJL bits are
// +-1 as they stand.  Every term of the score and of the value sum is then a
// product of an exact +-1 matrix (built from the packed bits with one shift
// and one LOP3 per pair of elements) and a bf16 hi/lo split of q~, S q~ or
// the softmax weights, so the per-token dot products run on the tensor pipe
// (mma.sync m16n8k16, fp32 accumulate) without dequantizing anything.
//   K side:  C[token][head,piece] = sum_dim s_p[token][dim] * q~hi/lo[dim]
//   V side:  O[dim][head,piece]   = sum_tok s_p[tok][dim] * (w_p p ||v||)hi/lo
// All G query heads of a KV head share each streamed record (GQA).
#include <cuda_bf16.h>

#include <cmath>
#include <mutex>

#include "bitplane.cuh"
#include "encode_vec.cuh"
#include "tcgen05.cuh"
#include "tq_internal.h"

namespace {

using namespace tqdev;

constexpr int kD = 128;        // head dimension handled here
constexpr int kWarps = 4;      // warps per CTA
constexpr int kTile = 16;      // tokens per MMA tile
constexpr int kStages = 4;     // cp.async ring depth per warp
constexpr float kLazyRescale = 8.0f;  // log2 units of headroom before rescaling

struct DecodeParams {
  const uint8_t* k_codes;
  const uint8_t* k_signs;
  const float2* k_norms;
  const uint8_t* v_codes;
  const uint8_t* v_signs;
  const float2* v_norms;
  int64_t cache_stride;
  int64_t T;
  int64_t chunk;           // tokens per split (multiple of kTile)
  int n_splits;
  int n_slots;             // partial records per head: n_splits, then one per window chunk
  const uint32_t* qfrag;   // [BH][MG][2 NT][32][2]: int8 digits of the key-side B operand
  const float4* kconst;    // [BH][8]: (2^-E code, code constant, 2^-E sign, sign constant) per head
  float* partial;          // [BH][n_slots][G][2 + 2 kD]
  float score_scale;       // softmax scale * log2(e)
  float qjl;               // sqrt(pi/2) / m
  float walsh_k[4];
  float walsh_v[4];
  uint32_t one_h, one_b;   // kOneH2 / kOneB2, passed at run time (see bit_select)
  const int32_t* seq_lens; // [B] tokens of each sequence (<= T), or null: all T
  int Hkv;
  int append;              // the preceding launch writes each sequence's last record: no copy before its end
  // NSN record mode ([NSNQuant] §1): s1 of every record (same indexing as the
  // norms) and <q', o_k> per query head ([BH][8], from q-prep)
  const float* k_s1;
  const float* v_s1;
  const float* qo;
};

// Floats of one partial record: m, l, O_code [kD], O_z [kD], and for the NSN
// mode sum_t p_t s1v_t and a pad.
template <bool NSN>
constexpr int partial_rec() { return 2 + 2 * kD + (NSN ? 2 : 0); }


// Key-side MMA groups of the split kernel (m16n8k32, u8 bits x s8 query
// digits).  A group covers 32 K elements per 16 tokens: with two Walsh planes
// a group takes byte position j (0..7) of one 32-coordinate word of each
// plane (one AND each: bits j, j+8, j+16, j+24 at weight 2^j); a single
// plane (1-bit codes, the sign plane) takes nibble position j (0..3) of the
// word and of the word shifted right by four.  CODE groups for the code
// planes, SIGN for the QJL signs.
template <int BITS>
struct KeyGroups {
  static constexpr int P = Planes<BITS>::P;            // Walsh planes
  static constexpr int CODE = BITS == 1 ? 4 : 8 * (P / 2);
  static constexpr int SIGN = 4;
  static constexpr int MG = CODE + SIGN;
};

struct WalshWeights {
  float w[4];
};

// Shared-memory position of the 16-byte chunk `part` (code plane) of token
// `tok`'s codes.  With 2-bit codes (two chunks per token) the chunks of tokens
// 4..7 (mod 8) are swapped so that the key side's word reads are free of bank
// conflicts.
template <int BITS>
__device__ __forceinline__ int code_chunk(int tok, int part) {
  if constexpr (BITS == 2) return tok * 2 + (part ^ ((tok >> 2) & 1));
  else return tok * BITS + part;
}

// Fast Walsh-Hadamard transform (Sylvester order, unnormalised) of one kD
// vector per group of kD threads, thread i of the group holding coordinate i:
// five stages by warp shuffles, the two across warps through the group's row
// of shared memory `buf`.  All groups of the block run it together.
__device__ __forceinline__ void fwht_group(float& v, int i, float* buf) {
  const int lane = i & 31;
#pragma unroll
  for (int bit = 1; bit < 32; bit <<= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, v, bit);
    v = (lane & bit) ? o - v : v + o;
  }
#pragma unroll
  for (int bit = 32; bit < kD; bit <<= 1) {
    __syncthreads();
    buf[i] = v;
    __syncthreads();
    const float o = buf[i ^ bit];
    v = (i & bit) ? o - v : v + o;
  }
}

template <int BITS, int G, bool NSN>
__global__ void __launch_bounds__(kWarps * 32, G <= 4 ? 3 : 1) decode_split_kernel(DecodeParams p) {
  constexpr int NT = (2 * G + 7) / 8;
  constexpr int P = Planes<BITS>::P;
  constexpr int CB = BITS * kD / 8;
  constexpr int SB = kD / 8;
  constexpr int HALF = kTile * (CB + SB + 8 + (NSN ? 4 : 0));   // codes, signs, norms (, s1) of one side
  constexpr int STAGE = 2 * HALF;
  constexpr int S1OFF = kTile * (CB + SB + 8);
  constexpr int CCH = kTile * CB / 16;
  extern __shared__ __align__(16) uint8_t smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int bh = blockIdx.y;
  const int split = blockIdx.x;
  const uint32_t one_b = p.one_b;
  // this sequence's length: T, or its own entry of seq_lens (a value outside
  // 0..T makes every output of the sequence NaN)
  int64_t T_seq = p.T;
  bool bad_len = false;
  if (p.seq_lens) {
    const int64_t v = p.seq_lens[bh / p.Hkv];
    bad_len = v < 0 || v > p.T;
    T_seq = bad_len ? 0 : v;
  }
  const int64_t t_begin = static_cast<int64_t>(split) * p.chunk;
  const int64_t t_end = min(T_seq, t_begin + p.chunk);
  const int n_tiles = t_end > t_begin ? static_cast<int>((t_end - t_begin + kTile - 1) / kTile) : 0;
  const int my_count = n_tiles > warp ? (n_tiles - warp + kWarps - 1) / kWarps : 0;
  const int64_t seq = static_cast<int64_t>(bh) * p.cache_stride;
  uint8_t* my_stages = smem + warp * kStages * STAGE;

  // Each lane copies 16-byte chunks of the tile's K and V codes, signs and
  // norms into the warp's stage (cp.async, a 4-stage ring per warp); rows past
  // the tile's last token are zero-filled.
  auto tile_nv = [&](int i) {
    const int64_t t0 = t_begin + static_cast<int64_t>(warp + kWarps * i) * kTile;
    return static_cast<int>(t_end - t0 < kTile ? t_end - t0 : kTile);
  };
  const int sg_side = lane >> 4, sg_c = lane & 15;
  const int nm_side = (lane >> 3) & 1, nm_c = lane & 7;
  // Per-lane copy plan of a full tile: sources advance by kWarps tiles per
  // issue, destinations are fixed offsets within a stage.
  constexpr int CIT = (CCH + 31) / 32;
  const int64_t tok0 = seq + t_begin + static_cast<int64_t>(warp) * kTile;
  const uint8_t* src_code[2][CIT];
  uint32_t dst_code[2][CIT];
#pragma unroll
  for (int side = 0; side < 2; ++side)
#pragma unroll
    for (int k = 0; k < CIT; ++k) {
      const int c = lane + 32 * k;
      const int cc = c < CCH ? c : 0;
      src_code[side][k] = (side ? p.v_codes : p.k_codes) + tok0 * CB + cc * 16;
      dst_code[side][k] = side * HALF + code_chunk<BITS>(cc / BITS, cc % BITS) * 16;
    }
  const uint8_t* src_sign = (sg_side ? p.v_signs : p.k_signs) + tok0 * SB + sg_c * 16;
  const uint32_t dst_sign = sg_side * HALF + kTile * CB + sg_c * 16;
  const uint8_t* src_norm = reinterpret_cast<const uint8_t*>((nm_side ? p.v_norms : p.k_norms) + tok0) + nm_c * 16;
  const uint32_t dst_norm = nm_side * HALF + kTile * (CB + SB) + nm_c * 16;
  // NSN: lanes 16..23 copy the tile's s1 (four tokens per lane; keys, then values)
  const int s1_side = (lane >> 2) & 1, s1_c = lane & 3;
  const uint8_t* src_s1 = nullptr;
  if constexpr (NSN) src_s1 = reinterpret_cast<const uint8_t*>((s1_side ? p.v_s1 : p.k_s1) + tok0) + s1_c * 16;
  const uint32_t dst_s1 = s1_side * HALF + S1OFF + s1_c * 16;
  constexpr int64_t kStepTok = static_cast<int64_t>(kWarps) * kTile;
  const int64_t n_full = (t_end - t_begin) / kTile;   // full tiles of the split (t_end >= t_begin or none)
  const int my_full = t_end > t_begin && n_full > warp ? static_cast<int>((n_full - warp + kWarps - 1) / kWarps) : 0;
  auto issue = [&](int i) {
    if (i < my_full) {
      uint8_t* stg = my_stages + (i % kStages) * STAGE;
      const int64_t adv = kStepTok * i;
#pragma unroll
      for (int side = 0; side < 2; ++side)
#pragma unroll
        for (int k = 0; k < CIT; ++k)
          if (lane + 32 * k < CCH) cp_async16(stg + dst_code[side][k], src_code[side][k] + adv * CB, 16);
      cp_async16(stg + dst_sign, src_sign + adv * SB, 16);
      if (lane < 16) cp_async16(stg + dst_norm, src_norm + adv * 8, 16);
      if constexpr (NSN) {
        if (lane >= 16 && lane < 24) cp_async16(stg + dst_s1, src_s1 + adv * 4, 16);
      }
    } else if (i < my_count) {
      const int64_t t0 = seq + t_begin + static_cast<int64_t>(warp + kWarps * i) * kTile;
      const int nv = tile_nv(i);
      uint8_t* stg = my_stages + (i % kStages) * STAGE;
#pragma unroll
      for (int side = 0; side < 2; ++side) {
        const uint8_t* src = (side ? p.v_codes : p.k_codes) + t0 * CB;
#pragma unroll
        for (int c = lane; c < CCH; c += 32) {
          const int tok = c / BITS, part = c % BITS;
          cp_async16(stg + side * HALF + code_chunk<BITS>(tok, part) * 16, tok < nv ? src + c * 16 : src,
                     tok < nv ? 16 : 0);
        }
      }
      {
        const uint8_t* src = (sg_side ? p.v_signs : p.k_signs) + t0 * SB;
        cp_async16(stg + sg_side * HALF + kTile * CB + sg_c * 16, sg_c < nv ? src + sg_c * 16 : src, sg_c < nv ? 16 : 0);
      }
      if (lane < 16) {
        const float2* src = (nm_side ? p.v_norms : p.k_norms) + t0;
        const int bytes = max(0, min(16, (nv - 2 * nm_c) * 8));
        cp_async16(stg + nm_side * HALF + kTile * (CB + SB) + nm_c * 16, bytes ? src + 2 * nm_c : src, bytes);
      }
      if constexpr (NSN) {
        if (lane >= 16 && lane < 24) {
          const float* src = (s1_side ? p.v_s1 : p.k_s1) + t0;
          const int bytes = max(0, min(16, (nv - 4 * s1_c) * 4));
          cp_async16(stg + s1_side * HALF + S1OFF + s1_c * 16, bytes ? src + 4 * s1_c : src, bytes);
        }
      }
    }
    cp_async_commit();
  };

  // The first tiles of the cache do not depend on the q-prep launch: start
  // their copies, then wait for q-prep's outputs (programmatic dependent
  // launch; a no-op when launched without it).
  if (!p.append) {
#pragma unroll 1
    for (int i = 0; i < kStages - 1; ++i) issue(i);
  }
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  if (p.append) {
#pragma unroll 1
    for (int i = 0; i < kStages - 1; ++i) issue(i);
  }

  // The key side's B operand (int8 digits of the query, one set of
  // fragments per MMA group and n-tile) in shared memory, read at each MMA;
  // the per-head scales and constants in registers.
  constexpr int MG = KeyGroups<BITS>::MG;
  constexpr int NTK = 2 * NT;
  // fp32x2 (two rows or two tokens per instruction, the same roundings) for
  // the key-side recombination and the softmax, and for the value weights:
  // chosen per instance by measurement of the split launch (Llama-8B-shaped
  // layer at G = 4, the 70B-shaped slice at G = 8): 2 bits G 4 the same with
  // the first, 4 % slower with the second; 3 bits G 4 3.6 % faster with the
  // second alone, slower with the first; 2 bits G 8 2.6 % faster with both;
  // 1 bit G 4 1 % slower with the first
  constexpr bool kPackKS = BITS == 2;
  constexpr bool kPackV = BITS == 3 || G == 8;
  __shared__ uint2 s_qf[MG][NTK][32];
  float4 kc[NT];
  float qo[NT];   // NSN: score_scale <q', o_k> of head tig + 4 nt
  {
    const uint2* src = reinterpret_cast<const uint2*>(p.qfrag) + static_cast<size_t>(bh) * (MG * NTK * 32);
    for (int i = threadIdx.x; i < MG * NTK * 32; i += blockDim.x) (&s_qf[0][0][0])[i] = src[i];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      // per-head scale and constant of the code sum and of the sign sum, with
      // the softmax scale (and the QJL constant for the signs) folded in
      const int h = tig + 4 * nt;
      float4 c = h < G ? p.kconst[static_cast<size_t>(bh) * 8 + h] : make_float4(0.f, 0.f, 0.f, 0.f);
      const float zs = p.qjl * p.score_scale;
      kc[nt] = make_float4(c.x * p.score_scale, c.y * p.score_scale, c.z * zs, c.w * zs);
      if constexpr (NSN) qo[nt] = h < G ? p.qo[static_cast<size_t>(bh) * 8 + h] * p.score_scale : 0.f;
    }
    __syncthreads();
  }
  float accC[NT][8][4], accZ[NT][8][4];
  float m_run[NT], l_run[NT];
  float sbc[NT], sbz[NT], s1sum[NT];   // s1sum: NSN, sum_t p_t s1v_t of this lane's tokens
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt] = -INFINITY;
    l_run[nt] = 0.f;
    sbc[nt] = sbz[nt] = s1sum[nt] = 0.f;
#pragma unroll
    for (int rb = 0; rb < 8; ++rb)
#pragma unroll
      for (int r = 0; r < 4; ++r) accC[nt][rb][r] = accZ[nt][rb][r] = 0.f;
  }
  const float piece_m = (gid & 1) ? 1.f : 0.f;   // this lane feeds the hi (0) or lo (1) piece
  // ---- K side of one tile: logits of tokens gid, gid + 8 for head tig + 4 nt.
  // m16n8k32 u8 x s8 products into int32: rows are the 16 tokens, K runs over
  // (plane, coordinate) slots, the columns are (head, digit); each A register
  // is one AND of a plane word (see KeyGroups), so every product is exact and
  // the four digit columns of a head recombine in fp32 (each column stays
  // below 2^22 in magnitude, where the float conversion is exact).
  auto k_side = [&](const uint8_t* stg, int nv, float (&logit)[NT][2]) {
    const uint8_t* kcd = stg;
    const uint32_t* ks = reinterpret_cast<const uint32_t*>(stg + kTile * CB);
    const float2* kn = reinterpret_cast<const float2*>(stg + kTile * (CB + SB));
    uint32_t wk[2][P], wz[2];
    float2 knorm[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int tok = gid + 8 * e;
      uint32_t raw[BITS];
#pragma unroll
      for (int k = 0; k < BITS; ++k)
        raw[k] = reinterpret_cast<const uint32_t*>(kcd + code_chunk<BITS>(tok, k) * 16)[tig];
      Planes<BITS>::make(raw, wk[e]);
      wz[e] = ks[tok * (SB / 4) + tig];
      knorm[e] = kn[tok];
    }
    int accc[NTK][4], accs[NTK][4];
#pragma unroll
    for (int n = 0; n < NTK; ++n)
#pragma unroll
      for (int r = 0; r < 4; ++r) accc[n][r] = accs[n][r] = kBiasedZero;   // every column stays below 2^22
    if constexpr (BITS == 1) {
      const uint32_t w4[2] = {wk[0][0] >> 4, wk[1][0] >> 4};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t M = 0x01010101u << j;
        const uint32_t a[4] = {wk[0][0] & M, wk[1][0] & M, w4[0] & M, w4[1] & M};
#pragma unroll
        for (int n = 0; n < NTK; ++n) {
          const uint2 b = s_qf[j][n][lane];
          mma_u8s8(accc[n], a, b.x, b.y);
        }
      }
    } else {
#pragma unroll
      for (int pr = 0; pr < P / 2; ++pr)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t M = 0x01010101u << j;
          const uint32_t a[4] = {wk[0][2 * pr] & M, wk[1][2 * pr] & M, wk[0][2 * pr + 1] & M, wk[1][2 * pr + 1] & M};
#pragma unroll
          for (int n = 0; n < NTK; ++n) {
            const uint2 b = s_qf[pr * 8 + j][n][lane];
            mma_u8s8(accc[n], a, b.x, b.y);
          }
        }
    }
    {
      const uint32_t z4[2] = {wz[0] >> 4, wz[1] >> 4};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t M = 0x01010101u << j;
        const uint32_t a[4] = {wz[0] & M, wz[1] & M, z4[0] & M, z4[1] & M};
#pragma unroll
        for (int n = 0; n < NTK; ++n) {
          const uint2 b = s_qf[KeyGroups<BITS>::CODE + j][n][lane];
          mma_u8s8(accs[n], a, b.x, b.y);
        }
      }
    }
    if constexpr (kPackKS) {
      // both rows (tokens gid, gid + 8) at once on fp32x2 instructions
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int c0[4] = {accc[2 * nt][0], accc[2 * nt][1], accc[2 * nt + 1][0], accc[2 * nt + 1][1]};
        const int c1[4] = {accc[2 * nt][2], accc[2 * nt][3], accc[2 * nt + 1][2], accc[2 * nt + 1][3]};
        const int z0[4] = {accs[2 * nt][0], accs[2 * nt][1], accs[2 * nt + 1][0], accs[2 * nt + 1][1]};
        const int z1[4] = {accs[2 * nt][2], accs[2 * nt][3], accs[2 * nt + 1][2], accs[2 * nt + 1][3]};
        const float2 code = __ffma2_rn(digits_to_float2(c0, c1), make_float2(kc[nt].x, kc[nt].x),
                                       make_float2(-kc[nt].y, -kc[nt].y));
        const float2 sgn = __ffma2_rn(digits_to_float2(z0, z1), make_float2(kc[nt].z, kc[nt].z),
                                      make_float2(-kc[nt].w, -kc[nt].w));
        float2 l = __ffma2_rn(make_float2(knorm[0].x, knorm[1].x), code,
                              __fmul2_rn(make_float2(knorm[0].y, knorm[1].y), sgn));
        if constexpr (NSN) {
          const float* s1 = reinterpret_cast<const float*>(stg + S1OFF);
          l = __ffma2_rn(make_float2(s1[gid], s1[gid + 8]), make_float2(qo[nt], qo[nt]), l);
        }
        logit[nt][0] = gid < nv ? l.x : -INFINITY;
        logit[nt][1] = gid + 8 < nv ? l.y : -INFINITY;
      }
    } else {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float code = fmaf(digits_to_float(accc[2 * nt][2 * e], accc[2 * nt][2 * e + 1],
                                                  accc[2 * nt + 1][2 * e], accc[2 * nt + 1][2 * e + 1]),
                                  kc[nt].x, -kc[nt].y);
          const float sgn = fmaf(digits_to_float(accs[2 * nt][2 * e], accs[2 * nt][2 * e + 1],
                                                 accs[2 * nt + 1][2 * e], accs[2 * nt + 1][2 * e + 1]),
                                 kc[nt].z, -kc[nt].w);
          float l = fmaf(knorm[e].x, code, knorm[e].y * sgn);
          if constexpr (NSN) l = fmaf(reinterpret_cast<const float*>(stg + S1OFF)[gid + 8 * e], qo[nt], l);
          logit[nt][e] = gid + 8 * e < nv ? l : -INFINITY;
        }
      }
    }
  };
  // 2^x of the softmax: the hardware approximation for 1- and 2-bit codes; the
  // 3-bit instance measured faster with the library function (0.383 against
  // 0.395 ms per Llama-8B-shaped layer), so it keeps it
  auto softmax_exp2 = [](float x) { return BITS == 3 ? exp2f(x) : exp2_approx(x); };
  // ---- online softmax: new running max (rescaling what is accumulated) and p
  auto softmax = [&](const float (&logit)[NT][2], float (&prob)[NT][2]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float mx = fmaxf(logit[nt][0], logit[nt][1]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const bool need = mx > m_run[nt] + kLazyRescale;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? softmax_exp2(m_run[nt] - mx) : 1.f;
        const float alpha_b = __shfl_sync(0xffffffffu, alpha, gid >> 1);
        l_run[nt] *= alpha;
        sbc[nt] *= alpha_b;
        sbz[nt] *= alpha_b;
        if constexpr (NSN) s1sum[nt] *= alpha_b;
#pragma unroll
        for (int rb = 0; rb < 8; ++rb)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            accC[nt][rb][r] *= alpha;
            accZ[nt][rb][r] *= alpha;
          }
        if (need) m_run[nt] = mx;
      }
      if constexpr (kPackKS) {
        const float2 x = __fadd2_rn(make_float2(logit[nt][0], logit[nt][1]), make_float2(-m_run[nt], -m_run[nt]));
        prob[nt][0] = softmax_exp2(x.x);
        prob[nt][1] = softmax_exp2(x.y);
        l_run[nt] += prob[nt][0] + prob[nt][1];
      } else {
#pragma unroll
        for (int e = 0; e < 2; ++e) prob[nt][e] = softmax_exp2(logit[nt][e] - m_run[nt]);
        l_run[nt] += prob[nt][0] + prob[nt][1];
      }
    }
  };

  // ---- V side of one tile with its probabilities
  auto v_side = [&](const uint8_t* stg, const float (&prob)[NT][2], int nv) {
    const uint8_t* vcd = stg + HALF;
    const uint8_t* vs = vcd + kTile * CB;
    const float2* vn = reinterpret_cast<const float2*>(vcd + kTile * (CB + SB));
    const int tk[4] = {2 * tig, 2 * tig + 1, 2 * tig + 8, 2 * tig + 9};
    // Transposing matrix loads: an 8 x 8 matrix of 16-bit elements whose row r
    // is the 16-byte plane (or sign) row of token r of a group of eight; the
    // transposed load hands lane (g, t) half-word g (coordinates 16g..16g+15)
    // of tokens 2t and 2t + 1 in one register, the pair a bit-select turns
    // into the two K elements of the value operand.  Lane l addresses row
    // l % 8 of matrix l / 8.
    uint32_t x01[P], x23[P], z01, z23;
    {
      uint32_t r01[BITS], r23[BITS];
      const int mi = lane >> 3, rr = lane & 7;
      const uint32_t vbase = tqtc::smem_u32(vcd), sbase = tqtc::smem_u32(vs);
      const uint32_t code_row = vbase + static_cast<uint32_t>(code_chunk<BITS>(rr + 8 * (mi & 1), mi >> 1) * 16);
      const uint32_t sign_row = sbase + static_cast<uint32_t>((rr + 8 * (mi & 1)) * SB);
      if constexpr (BITS == 1) {
        ldsm_x4_trans(r01[0], r23[0], z01, z23, mi < 2 ? code_row : sign_row);
      } else if constexpr (BITS == 2) {
        ldsm_x4_trans(r01[0], r23[0], r01[1], r23[1], code_row);
        ldsm_x2_trans(z01, z23, sign_row);
      } else {
        ldsm_x4_trans(r01[0], r23[0], r01[1], r23[1], code_row);
        ldsm_x4_trans(r01[2], r23[2], z01, z23,
                      mi < 2 ? vbase + static_cast<uint32_t>(code_chunk<BITS>(rr + 8 * mi, 2) * 16) : sign_row);
      }
      Planes<BITS>::make(r01, x01);
      Planes<BITS>::make(r23, x23);
    }
    uint32_t xs01[P], xs23[P];
#pragma unroll
    for (int q = 0; q < P; ++q) {
      xs01[q] = x01[q] << 8;
      xs23[q] = x23[q] << 8;
    }
    const uint32_t zs01 = z01 << 8, zs23 = z23 << 8;
    float2 vnorm[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) vnorm[j] = vn[tk[j]];
    const int srcA = (2 * tig) * 4 + (gid >> 1);
    const int srcB = (2 * tig + 1) * 4 + (gid >> 1);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pt[4];
      pt[0] = __shfl_sync(0xffffffffu, prob[nt][0], srcA);
      pt[2] = __shfl_sync(0xffffffffu, prob[nt][1], srcA);
      pt[1] = __shfl_sync(0xffffffffu, prob[nt][0], srcB);
      pt[3] = __shfl_sync(0xffffffffu, prob[nt][1], srcB);
      uint32_t bc[P][2], bz[2];
      float wv[4], wr[4];
      if constexpr (kPackV) {
#pragma unroll
        for (int j = 0; j < 4; j += 2) {   // rows past the tile's last token: p = 0, zero-filled norms
          const float2 pp = make_float2(pt[j], pt[j + 1]);
          const float2 a = __fmul2_rn(pp, make_float2(vnorm[j].x, vnorm[j + 1].x));
          const float2 b = __fmul2_rn(pp, make_float2(vnorm[j].y, vnorm[j + 1].y));
          wv[j] = a.x;
          wv[j + 1] = a.y;
          wr[j] = b.x;
          wr[j + 1] = b.y;
        }
        // B operand: lanes of even gid feed RN(w), odd gid RN(w - RN(w)), both
        // as bf16 pairs: one paired conversion, an FFMA by piece_m in {0, 1},
        // one paired conversion out (|w - hi - lo| <= 2^-17 |w|).
        const float2 npm = make_float2(-piece_m, -piece_m);
        auto pair2 = [&](float2 w) -> uint32_t {
          __nv_bfloat162 h = __floats2bfloat162_rn(w.x, w.y);
          const uint32_t hb = *reinterpret_cast<uint32_t*>(&h);
          const float2 r = __ffma2_rn(npm, make_float2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xFFFF0000u)), w);
          __nv_bfloat162 rb = __floats2bfloat162_rn(r.x, r.y);
          return *reinterpret_cast<uint32_t*>(&rb);
        };
#pragma unroll
        for (int pl = 0; pl < P; ++pl) {
          const float2 wp = make_float2(p.walsh_v[pl], p.walsh_v[pl]);
          bc[pl][0] = pair2(__fmul2_rn(wp, make_float2(wv[0], wv[1])));
          bc[pl][1] = pair2(__fmul2_rn(wp, make_float2(wv[2], wv[3])));
        }
        bz[0] = pair2(make_float2(wr[0], wr[1]));
        bz[1] = pair2(make_float2(wr[2], wr[3]));
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          wv[j] = pt[j] * vnorm[j].x;   // rows past the tile's last token: p = 0, zero-filled norms
          wr[j] = pt[j] * vnorm[j].y;
        }
        // B operand: lanes of even gid feed RN(w), odd gid RN(w - RN(w)), both
        // as bf16 pairs: one paired conversion, an FFMA by piece_m in {0, 1},
        // one paired conversion out (|w - hi - lo| <= 2^-17 |w|).
        auto pair2 = [&](float a, float b) -> uint32_t {
          __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
          const uint32_t hb = *reinterpret_cast<uint32_t*>(&h);
          const float ha = __uint_as_float(hb << 16), hbf = __uint_as_float(hb & 0xFFFF0000u);
          __nv_bfloat162 r = __floats2bfloat162_rn(fmaf(-piece_m, ha, a), fmaf(-piece_m, hbf, b));
          return *reinterpret_cast<uint32_t*>(&r);
        };
#pragma unroll
        for (int pl = 0; pl < P; ++pl) {
          bc[pl][0] = pair2(p.walsh_v[pl] * wv[0], p.walsh_v[pl] * wv[1]);
          bc[pl][1] = pair2(p.walsh_v[pl] * wv[2], p.walsh_v[pl] * wv[3]);
        }
        bz[0] = pair2(wr[0], wr[1]);
        bz[1] = pair2(wr[2], wr[3]);
      }
      // unrounded weight sums for the offset mu_p sum B (hi + lo differ from
      // w by at most 2^-17 |w|, far inside the output tolerance)
      sbc[nt] += (wv[0] + wv[1]) + (wv[2] + wv[3]);
      sbz[nt] += (wr[0] + wr[1]) + (wr[2] + wr[3]);
      if constexpr (NSN) {
        const float* vs1 = reinterpret_cast<const float*>(vcd + S1OFF);   // zero-filled past the tile's end
#pragma unroll
        for (int j = 0; j < 4; ++j) s1sum[nt] = fmaf(pt[j], vs1[tk[j]], s1sum[nt]);
      }
#pragma unroll
      for (int rb = 0; rb < 8; ++rb) {
#pragma unroll
        for (int pl = 0; pl < P; ++pl) {
          const uint32_t a[4] = {bit_pair_b(x01[pl], xs01[pl], 2 * rb, one_b),
                                 bit_pair_b(x01[pl], xs01[pl], 2 * rb + 1, one_b),
                                 bit_pair_b(x23[pl], xs23[pl], 2 * rb, one_b),
                                 bit_pair_b(x23[pl], xs23[pl], 2 * rb + 1, one_b)};
          mma_bf16(accC[nt][rb], a, bc[pl][0], bc[pl][1]);
        }
        const uint32_t a[4] = {bit_pair_b(z01, zs01, 2 * rb, one_b), bit_pair_b(z01, zs01, 2 * rb + 1, one_b),
                               bit_pair_b(z23, zs23, 2 * rb, one_b), bit_pair_b(z23, zs23, 2 * rb + 1, one_b)};
        mma_bf16(accZ[nt][rb], a, bz[0], bz[1]);
      }
    }
  };
  // Pipelined order: the key side of tile i and the value side of tile i - 1
  // share one loop body (for G = 8 this fits the register file because the
  // query fragments are in shared memory).
  {
    float prob_prev[NT][2];
    const uint8_t* stg_prev = my_stages;
    int nv_prev = 0;
    if (my_count > 0) {
      cp_async_wait<kStages - 2>();
      __syncwarp();
      float logit[NT][2];
      nv_prev = tile_nv(0);
      k_side(my_stages, nv_prev, logit);
      softmax(logit, prob_prev);
      issue(kStages - 1);   // stage kStages-1 is still unused
    }
#pragma unroll 1
    for (int i = 1; i < my_count; ++i) {
      cp_async_wait<kStages - 2>();
      __syncwarp();
      const uint8_t* stg = my_stages + (i % kStages) * STAGE;
      const int nv = tile_nv(i);
      float logit[NT][2];
      k_side(stg, nv, logit);             // independent of the V side below
      v_side(stg_prev, prob_prev, nv_prev);
      softmax(logit, prob_prev);
      stg_prev = stg;
      nv_prev = nv;
      __syncwarp();
      issue(i + kStages - 1);             // into the stage of tile i - 1
    }
    if (my_count > 0) v_side(stg_prev, prob_prev, nv_prev);
  }
  cp_async_wait<0>();
  if (bad_len) {   // a finite max keeps the NaN sum from being dropped by the merges
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m_run[nt] = 0.f;
      l_run[nt] = __int_as_float(0x7fc00000);
    }
  }
  __syncthreads();

  constexpr int REC = partial_rec<NSN>();
  float* mbuf = reinterpret_cast<float*>(smem);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = tig + 4 * nt;
    float l = l_run[nt];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    float bc_sum = sbc[nt], bz_sum = sbz[nt];
    bc_sum += __shfl_xor_sync(0xffffffffu, bc_sum, 1);
    bc_sum += __shfl_xor_sync(0xffffffffu, bc_sum, 2);
    bz_sum += __shfl_xor_sync(0xffffffffu, bz_sum, 1);
    bz_sum += __shfl_xor_sync(0xffffffffu, bz_sum, 2);
    // column sums of the fed B over the split: every lane holds the full
    // weights of its tokens, so one lane of the head's (hi, lo) pair suffices;
    // the code operand of plane p carried walsh_v[p] w
    float wsum = 0.f;
#pragma unroll
    for (int pl = 0; pl < P; ++pl) wsum += p.walsh_v[pl];
    const float SBc = __shfl_sync(0xffffffffu, bc_sum, 8 * tig) * wsum;
    const float SBz = __shfl_sync(0xffffffffu, bz_sum, 8 * tig);
    float S1v = 0.f;
    if constexpr (NSN) {   // the same reduction as the weight sums
      float v = s1sum[nt];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      S1v = __shfl_sync(0xffffffffu, v, 8 * tig);
    }
    if (h < G) {
      float* dst = mbuf + (warp * G + h) * REC;
      if (gid == 0) {
        dst[0] = m_run[nt];
        dst[1] = l;
        if constexpr (NSN) {
          dst[2 + 2 * kD] = S1v;
          dst[3 + 2 * kD] = 0.f;
        }
      }
#pragma unroll
      for (int rb = 0; rb < 8; ++rb) {
        const int d0 = 16 * gid + 2 * rb;
        const int p0 = slot_pos(2 * rb), p1 = slot_pos(2 * rb + 1);
        const float mu0 = 0.5f * (pos_v0_b(p0) + pos_v1_b(p0)), is0 = 2.f / (pos_v1_b(p0) - pos_v0_b(p0));
        const float mu1 = 0.5f * (pos_v0_b(p1) + pos_v1_b(p1)), is1 = 2.f / (pos_v1_b(p1) - pos_v0_b(p1));
        dst[2 + d0] = (accC[nt][rb][0] + accC[nt][rb][1] - mu0 * SBc) * is0;
        dst[2 + d0 + 1] = (accC[nt][rb][2] + accC[nt][rb][3] - mu1 * SBc) * is1;
        dst[2 + kD + d0] = (accZ[nt][rb][0] + accZ[nt][rb][1] - mu0 * SBz) * is0;
        dst[2 + kD + d0 + 1] = (accZ[nt][rb][2] + accZ[nt][rb][3] - mu1 * SBz) * is1;
      }
    }
  }
  __syncthreads();
  float* out = p.partial + (static_cast<size_t>(bh) * p.n_slots + split) * G * REC;
  for (int idx = threadIdx.x; idx < G * REC; idx += blockDim.x) {
    const int h = idx / REC, k = idx % REC;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mbuf[(w * G + h) * REC]);
    float acc = 0.f;
    if (k == 0) {
      acc = M;
    } else if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = mbuf[(w * G + h) * REC];
        if (mw != -INFINITY) acc = fmaf(exp2f(mw - M), mbuf[(w * G + h) * REC + k], acc);
      }
    }
    out[idx] = acc;
  }
}


// One block of G groups of kD threads per (sequence b, KV head); group h is
// query head h of the group, thread i of it coordinate i: RoPE, q~ = Pi q,
// s = S q~, then the int8 B fragments of the split kernel's key side.  The product S q~
// is split by columns of S instead of by heads: group g holds columns
// [g kD/G, (g + 1) kD/G) of row i of S in registers (loaded before the wait
// for q, so the loads overlap the previous launch) and forms the partial sums
// of all G heads over them; the G partials meet in shared memory.
// Arguments of the query preparation (one block of G x kD threads per
// sequence bh = b * Hkv + kv).
template <typename T>
struct QPrepArgs {
  const T* q;              // [B Hq][kD]; query head h of the group is row bh * G + h
  const int64_t* q_pos;    // [B]
  int Hkv;
  const float* dsigns;
  const float* st;
  const float2* rope_hi;
  const float2* rope_lo;
  int64_t rope_max_pos;
  int rope;
  WalshWeights walsh;
  uint32_t* qfrag;
  float4* kconst;
  const float* o_k;        // NSN: the key shift o of each sequence [BH][kD] (or null)
  float* qo;               // NSN: <q', o_k> per query head [BH][8]
};

template <typename T, int G, int BITS>
__device__ __forceinline__ void qprep_body(const QPrepArgs<T>& a, int bh) {
  const T* __restrict__ q = a.q;
  const int64_t* __restrict__ q_pos = a.q_pos;
  const int Hkv = a.Hkv;
  const float* __restrict__ dsigns = a.dsigns;
  const float* __restrict__ st = a.st;
  const float2* __restrict__ rope_hi = a.rope_hi;
  const float2* __restrict__ rope_lo = a.rope_lo;
  const int64_t rope_max_pos = a.rope_max_pos;
  const int rope = a.rope;
  const WalshWeights& walsh = a.walsh;
  uint32_t* __restrict__ qfrag = a.qfrag;
  float4* __restrict__ kconst = a.kconst;
  constexpr int NT = (G + 3) / 4;
  constexpr int KS = kD / G;   // columns of S per group
  __shared__ __align__(16) float buf[G][kD];
  __shared__ __align__(16) float part[G][G][kD];   // [column group][head][i]
  __shared__ float red[2][G][2][kD / 32];
  const int tid = threadIdx.x, h = tid / kD, i = tid % kD, lane = tid & 31, wg = i >> 5;
  const int b = bh / Hkv;
  float scol[KS];
#pragma unroll
  for (int k = 0; k < KS; ++k) scol[k] = __ldg(st + (h * KS + k) * kD + i);
  // S belongs to the handle; q may come from the previous launch
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  float v;
  {
    const size_t at = (static_cast<size_t>(bh) * G + h) * kD + i;
    if constexpr (sizeof(T) == 4) v = q[at];
    else v = __bfloat162float(q[at]);
  }
  if (rope) {
    const int64_t pos = q_pos[b];
    buf[h][i] = v;
    __syncthreads();
    if (pos < 0 || pos >= rope_max_pos) {
      v = __int_as_float(0x7fc00000);
    } else {
      const int j = i & (kD / 2 - 1);
      const float2 a = rope_hi[(pos >> kRopeLoBits) * (kD / 2) + j];
      const float2 c = rope_lo[(pos & (kRopeLoRows - 1)) * (kD / 2) + j];
      const float cs = a.x * c.x - a.y * c.y, sn = a.y * c.x + a.x * c.y;
      const float x1 = buf[h][j], x2 = buf[h][j + kD / 2];
      v = i < kD / 2 ? x1 * cs - x2 * sn : x2 * cs + x1 * sn;
    }
  }
  // NSN: <q', o_k> of this head (q' after RoPE), summed over the group
  __shared__ float qsum[G][kD / 32];
  if (a.o_k) {
    float t = v * a.o_k[static_cast<size_t>(bh) * kD + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) qsum[h][wg] = t;
  }
  // q~ = H (D q) / sqrt(d)
  v *= dsigns[i];
  fwht_group(v, i, buf[h]);
  v *= rsqrtf(static_cast<float>(kD));
  __syncthreads();
  buf[h][i] = v;
  __syncthreads();
  // partial S q~ of every head over this group's columns of S
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < KS; ++k) acc = fmaf(scol[k], buf[hh][h * KS + k], acc);
    part[h][hh][i] = acc;
  }
  __syncthreads();
  float sv = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) sv += part[g][h][i];

  // Scatter into the int8 B fragments of the split kernel's key side.  The
  // key operand holds bit b of a plane at weight 2^j (j its position inside
  // its byte, or inside its nibble for the single-plane groups), so the value
  // that multiplies it is x 2^E / 2^j, x = 2 w_p q~_i for Walsh plane p and
  // x = 2 (S q~)_i for the sign plane (a 0/1 bit b stands for 2b - 1); E puts
  // max |x| just below 2^30, and the rounded value is cut into four balanced
  // signed bytes (digits).  Digit d of head h is column 2 (h % 4) + (d % 2) of
  // n-tile 2 (h / 4) + d / 2, so thread t of the split kernel holds all four
  // digits of head t (+ 4 per head group).
  constexpr int NTK = 2 * NT;
  constexpr int MG = KeyGroups<BITS>::MG;
  const int t = i >> 5, e = (i >> 3) & 3, j8 = i & 7;
  float mx[2] = {fabsf(v), fabsf(sv)};
#pragma unroll
  for (int ty = 0; ty < 2; ++ty) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx[ty] = fmaxf(mx[ty], __shfl_xor_sync(0xffffffffu, mx[ty], o));
    if (lane == 0) red[0][h][ty][wg] = mx[ty];
  }
  float csum = v, ssum = sv;   // sums over coordinates of q~ and S q~
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    csum += __shfl_xor_sync(0xffffffffu, csum, o);
    ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
  }
  if (lane == 0) {
    red[1][h][0][wg] = csum;
    red[1][h][1][wg] = ssum;
  }
  __syncthreads();
  float wmax = 0.f, wsum = 0.f;
#pragma unroll
  for (int pl = 0; pl < KeyGroups<BITS>::P; ++pl) {
    wmax = fmaxf(wmax, fabsf(walsh.w[pl]));
    wsum += walsh.w[pl];
  }
  int E[2];
#pragma unroll
  for (int ty = 0; ty < 2; ++ty) {
    const float m = fmaxf(fmaxf(red[0][h][ty][0], red[0][h][ty][1]), fmaxf(red[0][h][ty][2], red[0][h][ty][3])) *
                    (ty == 0 ? 2.f * wmax : 2.f);
    int ex = 0;
    if (m > 0.f && isfinite(m)) frexpf(m, &ex);   // m in [2^(ex-1), 2^ex)
    E[ty] = m > 0.f && isfinite(m) ? 30 - ex : 0;
  }
  uint8_t* frag = reinterpret_cast<uint8_t*>(qfrag);
  auto put = [&](int mg, int reg, int jj, float x, int ty) {
    // round(x 2^E / 2^jj), then four balanced digits
    int V = __float2int_rn(ldexpf(x, E[ty] - jj));
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      const int dg = ((V + 128) & 0xFF) - 128;
      V = (V - dg) >> 8;
      const int ntk = 2 * (h >> 2) + (d >> 1), g = 2 * (h & 3) + (d & 1);
      frag[((((static_cast<size_t>(bh) * MG + mg) * NTK + ntk) * 32 + 4 * g + t) * 2 + reg) * 4 + e] =
          static_cast<uint8_t>(dg);
    }
  };
  if constexpr (BITS == 1) {
    put(j8 & 3, j8 >> 2, j8 & 3, 2.f * walsh.w[0] * v, 0);
  } else {
#pragma unroll
    for (int pl = 0; pl < KeyGroups<BITS>::P; ++pl) put((pl >> 1) * 8 + j8, pl & 1, j8, 2.f * walsh.w[pl] * v, 0);
  }
  put(KeyGroups<BITS>::CODE + (j8 & 3), j8 >> 2, j8 & 3, 2.f * sv, 1);
  if constexpr (G < 4) {
    // columns of the absent heads of the first head group are zero
    for (int idx = tid; idx < MG * 2 * 32 * 2 * 4; idx += blockDim.x) {
      const int by = idx & 3, reg = (idx >> 2) & 1, ln = (idx >> 3) & 31, rest = idx >> 8;
      const int ntk = rest & 1, mg = rest >> 1;
      if ((ln >> 2) >= 2 * G)
        frag[((((static_cast<size_t>(bh) * MG + mg) * NTK + ntk) * 32 + ln) * 2 + reg) * 4 + by] = 0;
    }
  }
  if (i == 0) {
    const float cs = (red[1][h][0][0] + red[1][h][0][1]) + (red[1][h][0][2] + red[1][h][0][3]);
    const float ss = (red[1][h][1][0] + red[1][h][1][1]) + (red[1][h][1][2] + red[1][h][1][3]);
    kconst[static_cast<size_t>(bh) * 8 + h] = make_float4(ldexpf(1.f, -E[0]), wsum * cs, ldexpf(1.f, -E[1]), ss);
    if (a.o_k) a.qo[static_cast<size_t>(bh) * 8 + h] = (qsum[h][0] + qsum[h][1]) + (qsum[h][2] + qsum[h][3]);
  }
}

template <typename T, int G, int BITS>
__global__ void __launch_bounds__(kD * G) decode_qprep_kernel(const __grid_constant__ QPrepArgs<T> a) {
  qprep_body<T, G, BITS>(a, blockIdx.x);
}

// The decode step's append and query preparation in one launch: blocks
// 0..BH-1 prepare the queries (qprep_body); the others hold G groups of kD
// threads, each encoding one new row (encode_vec_core) into the record
// before the end of its sequence: keys (RoPE at the query's position) for
// vectors e < BH, values after.  [NSNQuant] §4 ("Résidus": quantize and
// append); [TurboESM] §3 (the record format).
struct AppendArgs {
  int BH;
  int64_t T;
  const int32_t* seq_lens;   // [B] or null: every sequence holds T tokens (the new one included)
  int64_t cache_stride;
  const float* k_o;          // NSN records: [BH][kD] shift of each sequence's keys (values: v_o), else null
  const float* v_o;
};

template <typename T, int G, int BITS>
__global__ void __launch_bounds__(kD * G) decode_prep_kernel(const __grid_constant__ QPrepArgs<T> a,
                                                            const __grid_constant__ AppendArgs ap,
                                                            const __grid_constant__ EncodeParams pk,
                                                            const __grid_constant__ EncodeParams pv) {
  if (static_cast<int>(blockIdx.x) < ap.BH) {
    qprep_body<T, G, BITS>(a, blockIdx.x);
    return;
  }
  __shared__ __align__(16) float gbuf[G][kD];
  __shared__ float gred[G][2][kD / 32];
  const int gi = threadIdx.x / kD, i = threadIdx.x % kD;
  const int64_t e = static_cast<int64_t>(blockIdx.x - ap.BH) * G + gi;
  asm volatile("griddepcontrol.wait;\n" ::: "memory");   // the cache may be read by the previous launch
  if (e >= 2 * static_cast<int64_t>(ap.BH)) return;       // uniform over the group
  const bool is_v = e >= ap.BH;
  const int64_t sq = is_v ? e - ap.BH : e;                 // sequence b * Hkv + kv
  const int b = static_cast<int>(sq / a.Hkv);
  const int64_t len = ap.seq_lens ? ap.seq_lens[b] : ap.T;
  if (len < 1 || len > ap.T) return;                       // nothing to append to (the decode gives NaN or zeros)
  const EncodeParams& p = is_v ? pv : pk;
  const int64_t rec = sq * ap.cache_stride + len - 1;
  const int64_t pos = p.rope ? a.q_pos[b] : 0;
  const float* o = is_v ? ap.v_o : ap.k_o;
  encode_vec_core<kD, BITS, T>(p, i, static_cast<const T*>(p.x) + sq * p.ld, rec, pos, gbuf[gi], gred[gi],
                               [gi] { asm volatile("bar.sync %0, %1;\n" ::"r"(1 + gi), "r"(kD) : "memory"); },
                               [&](int k) { return __ldg(p.st + k * kD + i); }, o ? o + sq * kD : nullptr);
}

// One block of G groups of kD threads per (sequence b, KV head); group h is
// query head h of the KV head, thread i of it coordinate i: log-sum-exp merge
// of the split partials, the QJL value correction sqrt(pi/2)/m S^T O_z, and
// Pi^T.  The product S^T O_z is split by rows of S instead of by heads: group
// g holds rows [g kD/G, (g + 1) kD/G) of column i of S in registers (loaded
// before the wait for the split kernel, so the loads overlap its tail) and
// forms the partial sums of all G heads over them; the G partials meet in
// shared memory.  The split weights f_s = 2^(m_s - M) of each head are formed
// by the first warp of its group and staged in shared memory (dynamic,
// n_splits * G floats), so each thread's sums over splits are plain loads.
//
// Partial records of sequence bh, part s, head h sit at
// partial + bh * bh_stride + s * part_stride + h * (2 + 2 kD): the split
// partials of one call, or the partials several calls (e.g. the ranks of a
// sequence-sharded decode) produced for the same heads.  With FINAL false the
// kernel stops after the log-sum-exp combination and writes the combined
// partial record (max, sum of weights, O_code, O_z) of each head to
// out[(bh G + h) (2 + 2 kD)], for a later merge with other such records.
template <int G, bool FINAL, bool NSN = false>
__global__ void __launch_bounds__(kD * G) decode_merge_kernel(const float* __restrict__ partial, int n_splits,
                                                             int64_t bh_stride, int64_t part_stride,
                                                             const float* __restrict__ s_mat,
                                                             const float* __restrict__ dsigns, float qjl,
                                                             float* __restrict__ out,
                                                             const float* __restrict__ v_o = nullptr) {
  static_assert(FINAL || !NSN, "NSN records merge into the output only");
  constexpr int REC = partial_rec<NSN>();
  constexpr int KS = kD / G;   // rows of S per group
  __shared__ __align__(16) float oz[G][kD];
  __shared__ __align__(16) float part[G][G][kD];   // [row group][head][i]
  __shared__ __align__(16) float buf[G][kD];
  __shared__ float Ls[G], Ms[G], S1s[G];
  extern __shared__ float fs[];   // [n_splits][G]
  const int tid = threadIdx.x, h = tid / kD, i = tid % kD, lane = tid & 31;
  const int bh = blockIdx.x;
  float scol[KS];
  if constexpr (FINAL) {
#pragma unroll
    for (int j = 0; j < KS; ++j) scol[j] = __ldg(s_mat + (h * KS + j) * kD + i);
  }
  asm volatile("griddepcontrol.wait;\n" ::: "memory");   // the split kernel's partials
  const float* base = partial + static_cast<size_t>(bh) * bh_stride + static_cast<size_t>(h) * REC;
  if (i < 32) {
    float M = -INFINITY;
    for (int s = lane; s < n_splits; s += 32) M = fmaxf(M, base[static_cast<size_t>(s) * part_stride]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float l = 0.f, s1 = 0.f;
    for (int s = lane; s < n_splits; s += 32) {
      const float* rec = base + static_cast<size_t>(s) * part_stride;
      const float ms = rec[0];
      const float f = (M == -INFINITY || ms == -INFINITY) ? 0.f : exp2f(ms - M);
      fs[s * G + h] = f;
      l = fmaf(f, rec[1], l);
      if constexpr (NSN) s1 = fmaf(f, rec[2 + 2 * kD], s1);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, o);
      if constexpr (NSN) s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    }
    if (lane == 0) {
      Ls[h] = l;
      Ms[h] = M;
      S1s[h] = s1;
    }
  }
  __syncthreads();
  float c = 0.f, z = 0.f;
#pragma unroll 4
  for (int s = 0; s < n_splits; ++s) {
    const float f = fs[s * G + h];
    const float* rec = base + static_cast<size_t>(s) * part_stride;
    c = fmaf(f, rec[2 + i], c);
    z = fmaf(f, rec[2 + kD + i], z);
  }
  if constexpr (!FINAL) {
    float* dst = out + (static_cast<size_t>(bh) * G + h) * REC;
    if (i == 0) {
      dst[0] = Ms[h];
      dst[1] = Ls[h];
    }
    dst[2 + i] = c;
    dst[2 + kD + i] = z;
    return;
  }
  oz[h][i] = z;
  __syncthreads();
  // partial S^T O_z of every head over this group's rows of S
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < KS; ++j) acc = fmaf(scol[j], oz[hh][h * KS + j], acc);
    part[h][hh][i] = acc;
  }
  __syncthreads();
  float corr = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) corr += part[g][h][i];
  // rotated-space value: O_code + sqrt(pi/2)/m S^T O_z, then Pi^T y = D H y / sqrt(d)
  float y = Ls[h] != 0.f ? (c + qjl * corr) / Ls[h] : 0.f;   // a NaN sum (a failed part) stays NaN
  fwht_group(y, i, buf[h]);
  float r = y * (dsigns[i] * rsqrtf(static_cast<float>(kD)));
  // NSN values: v_t = v'_t + s1v_t o_v, so the output gains o_v sum p s1v / l
  if constexpr (NSN) r = Ls[h] != 0.f ? fmaf(v_o[static_cast<size_t>(bh) * kD + i], S1s[h] / Ls[h], r) : r;
  out[(static_cast<size_t>(bh) * G + h) * kD + i] = r;
}

// (cos, sin) of pos * theta_j from the two RoPE tables: the angle of the
// coarse row pos >> kRopeLoBits plus that of the fine row pos mod kRopeLoRows.
__device__ __forceinline__ float2 rope_cs(const float2* __restrict__ rope_hi, const float2* __restrict__ rope_lo,
                                          int64_t pos, int j) {
  const float2 a = rope_hi[(pos >> kRopeLoBits) * (kD / 2) + j];
  const float2 c = rope_lo[(pos & (kRopeLoRows - 1)) * (kD / 2) + j];
  return make_float2(a.x * c.x - a.y * c.y, a.y * c.x + a.x * c.y);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x) {
  if constexpr (sizeof(T) == 4) return x;
  else return __bfloat162float(x);
}

constexpr int kWindowMax = 1024;   // tokens of a full-precision window
constexpr int kWinChunk = 32;      // window tokens per block, one partial record each

// The full-precision window ([NSNQuant] §4, "Résidus", after KIVI): the R most
// recent tokens of each sequence, kept as the model produced them, scored and
// summed exactly and written as split partials of their own, which the merge
// combines with the packed cache's partials by the same log-sum-exp rule.
// One block of four warps per (chunk of 32 window tokens, sequence b and KV
// head), for all G query heads of the KV head:
//  1. q' = RoPE(q, q_pos) in the original space (thread i: coordinate i).
//  2. Logits: warp w takes tokens w + 4u; lane l holds coordinates l + 32c
//     (c < 4), so both members of a RoPE pair (j, j + kD/2) sit in one lane;
//     token t gets RoPE at position T + t (after the packed part).  The key
//     and value rows of all of a warp's tokens are loaded at the start,
//     before the query is formed.
//  3. Softmax statistics of the chunk per head (max, then 2^(logit - max)
//     and their sum), one warp per head, one lane per token.
//  4. acc = sum_t w_t v_t in the original space: lane l of warp w sums
//     coordinates 4l .. 4l + 3 over the warp's tokens (vector loads), the four
//     warps' sums meet in shared memory; then y = Pi_V acc = H (D_V acc) /
//     sqrt(d) with the value handle's signs D_V, the rotated space the merge
//     applies Pi_V^T to.  The QJL half of the partial is zero.
template <typename TW, int G>
__global__ void __launch_bounds__(kD) decode_window_kernel(
    const void* __restrict__ q, int q_f32, const int64_t* __restrict__ q_pos, int Hkv, const TW* __restrict__ k_win,
    const TW* __restrict__ v_win, int64_t win_stride, int R, int64_t T_all, const int32_t* __restrict__ seq_lens,
    const float* __restrict__ v_dsigns,
    const float2* __restrict__ rope_hi, const float2* __restrict__ rope_lo, int64_t rope_max_pos, int rope,
    float score_scale, float* __restrict__ partial, int n_slots, int slot0) {
  constexpr int REC = 2 + 2 * kD;
  constexpr int TPW = kWinChunk / 4;   // tokens per warp
  __shared__ __align__(16) float qs[G][kD];
  __shared__ __align__(16) float red[4][G][kD];   // per-warp value sums (first: the raw query)
  __shared__ float lg[G][kWinChunk];              // logits, then weights
  __shared__ float stat[2][G];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y, b = bh / Hkv, chunk = blockIdx.x;
  const int t0 = chunk * kWinChunk;
  // the window follows this sequence's packed tokens; a length outside
  // 0..T_all makes the sequence's outputs NaN
  int64_t T = T_all;
  bool bad_len = false;
  if (seq_lens) {
    const int64_t v = seq_lens[b];
    bad_len = v < 0 || v > T_all;
    T = bad_len ? 0 : v;
  }
  const int n = min(kWinChunk, R - t0);   // >= 1: the host launches ceil(R / kWinChunk) chunks
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  // The key and value rows of this warp's tokens do not depend on the query:
  // their loads are issued first and overlap the query's RoPE below.
  const size_t row0 = static_cast<size_t>(bh) * win_stride + t0;
  float x[TPW][4], vv[TPW][4];
#pragma unroll
  for (int u = 0; u < TPW; ++u) {
    const int t = warp + 4 * u;
    const size_t row = row0 + (t < n ? t : 0);
    const TW* kr = k_win + row * kD;
#pragma unroll
    for (int c = 0; c < 4; ++c) x[u][c] = to_f32(kr[lane + 32 * c]);
    const TW* vr = v_win + row * kD + 4 * lane;
    if constexpr (sizeof(TW) == 4) {
      const float4 w = *reinterpret_cast<const float4*>(vr);
      vv[u][0] = w.x, vv[u][1] = w.y, vv[u][2] = w.z, vv[u][3] = w.w;
    } else {
      const uint2 w = *reinterpret_cast<const uint2*>(vr);
      vv[u][0] = __uint_as_float(w.x << 16), vv[u][1] = __uint_as_float(w.x & 0xFFFF0000u);
      vv[u][2] = __uint_as_float(w.y << 16), vv[u][3] = __uint_as_float(w.y & 0xFFFF0000u);
    }
  }
  // (cos, sin) of the keys' RoPE pairs j = lane and lane + 32, at position
  // T + t, below rope_max_pos for t < n (checked by the host)
  float2 kcs[TPW][2];
#pragma unroll
  for (int u = 0; u < TPW; ++u) {
    const int t = warp + 4 * u;
#pragma unroll
    for (int c = 0; c < 2; ++c)
      kcs[u][c] = rope && t < n ? rope_cs(rope_hi, rope_lo, T + t0 + t, lane + 32 * c) : make_float2(1.f, 0.f);
  }
  float* qraw = &red[0][0][0];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const size_t at = (static_cast<size_t>(bh) * G + h) * kD + tid;
    qraw[h * kD + tid] =
        q_f32 ? static_cast<const float*>(q)[at] : __bfloat162float(static_cast<const __nv_bfloat16*>(q)[at]);
  }
  __syncthreads();
  {
    const int j = tid & (kD / 2 - 1);
    float2 cs = make_float2(1.f, 0.f);
    bool bad = false;
    if (rope) {
      const int64_t pos = q_pos[b];
      bad = pos < 0 || pos >= rope_max_pos;
      if (!bad) cs = rope_cs(rope_hi, rope_lo, pos, j);
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v = qraw[h * kD + tid];
      if (rope) {
        const float x1 = qraw[h * kD + j], x2 = qraw[h * kD + j + kD / 2];
        v = bad ? __int_as_float(0x7fc00000) : (tid < kD / 2 ? x1 * cs.x - x2 * cs.y : x2 * cs.x + x1 * cs.y);
      }
      qs[h][tid] = v;
    }
  }
  __syncthreads();
  {
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
      const int t = warp + 4 * u;
      if (rope) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const float2 cs = kcs[u][c];
          const float x1 = x[u][c], x2 = x[u][c + 2];
          x[u][c] = x1 * cs.x - x2 * cs.y;
          x[u][c + 2] = x2 * cs.x + x1 * cs.y;
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) s = fmaf(qs[h][lane + 32 * c], x[u][c], s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) lg[h][t] = t < n ? s * score_scale : -INFINITY;
      }
    }
  }
  __syncthreads();
  for (int h = warp; h < G; h += 4) {
    const float s = lg[h][lane];
    float mx = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float e = exp2f(s - mx);
    lg[h][lane] = e;
    float l = e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      stat[0][h] = bad_len ? 0.f : mx;
      stat[1][h] = bad_len ? __int_as_float(0x7fc00000) : l;
    }
  }
  __syncthreads();
  {
    float acc[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
      const int t = warp + 4 * u;
      if (t < n) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float w = lg[h][t];
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[h][c] = fmaf(w, vv[u][c], acc[h][c]);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
      *reinterpret_cast<float4*>(&red[warp][h][4 * lane]) = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
  }
  __syncthreads();
  const float dsg = v_dsigns[tid];
  for (int h = 0; h < G; ++h) {
    float y = ((red[0][h][tid] + red[1][h][tid]) + (red[2][h][tid] + red[3][h][tid])) * dsg;
    fwht_group(y, tid, qs[0]);
    y *= rsqrtf(static_cast<float>(kD));
    float* rec = partial + ((static_cast<size_t>(bh) * n_slots + slot0 + chunk) * G + h) * REC;
    if (tid == 0) {
      rec[0] = stat[0][h];
      rec[1] = stat[1][h];
    }
    rec[2 + tid] = y;
    rec[2 + kD + tid] = 0.f;
  }
}

thread_local cudaEvent_t g_prof_begin = nullptr;
thread_local cudaEvent_t g_prof_end = nullptr;

struct SplitPlan {
  int n_splits;
  int64_t chunk;
};

SplitPlan plan_splits(int BH, int64_t T) {
  SplitPlan sp{1, kTile * kWarps};
  if (T <= 0) return sp;
  const int target = 148 * 8;
  int64_t ns = (target + BH - 1) / BH;
  const int64_t max_ns = (T + 255) / 256;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  int64_t chunk = (T + ns - 1) / ns;
  chunk = (chunk + kTile * kWarps - 1) / (kTile * kWarps) * (kTile * kWarps);
  sp.chunk = chunk;
  sp.n_splits = static_cast<int>((T + chunk - 1) / chunk);
  return sp;
}

// Key-side B fragments: [BH][MG][2 NT][32][2] u32, MG for the largest code
// (3 bits: 20 groups), NT = ceil(G / 4) head groups.
size_t frag_bytes(int BH, int G) {
  return static_cast<size_t>(BH) * KeyGroups<3>::MG * 2 * ((G + 3) / 4) * 32 * 2 * 4;
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

size_t kconst_bytes(int BH) { return static_cast<size_t>(BH) * 8 * sizeof(float4); }

// Sequences (batch x KV heads) of one call: the split kernel's grid has one
// row of blocks per sequence, and CUDA caps a grid's y extent at 65535.
constexpr int64_t kMaxSequences = 65535;

// Checks of the handles and sizes alone (no pointers), in the order the
// entry points report them: TQ_EINVAL for malformed sizes, TQ_EUNSUPPORTED
// for well-formed requests this library does not serve.
int check_decode_sizes(const tq_rotation* hk, const tq_rotation* hv, int B, int Hq, int Hkv, int64_t T) {
  if (!hk || !hv) return TQ_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || T < 0) return TQ_EINVAL;
  if (hk->d != hv->d || hk->m != hv->m) return TQ_EINVAL;
  if (static_cast<int64_t>(B) * Hkv > kMaxSequences) return TQ_EUNSUPPORTED;
  if (hk->d != kD || hk->m != kD) return TQ_EUNSUPPORTED;
  if (hk->kind != TQ_ROT_HADAMARD || hv->kind != TQ_ROT_HADAMARD) return TQ_EUNSUPPORTED;
  if (hk->bits != hv->bits) return TQ_EUNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return TQ_EUNSUPPORTED;
  return TQ_OK;
}

// Workspace bytes of one call; B * Hkv must already be within kMaxSequences.
size_t workspace_for(int B, int Hq, int Hkv, int64_t T, int R = 0) {
  const int G = Hq / Hkv;
  const int BH = B * Hkv;
  const SplitPlan sp = plan_splits(BH, T);
  const int slots = sp.n_splits + (R + kWinChunk - 1) / kWinChunk;
  return align256(frag_bytes(BH, G)) + align256(kconst_bytes(BH)) +
         align256(static_cast<size_t>(BH) * slots * G * partial_rec<true>() * sizeof(float)) +
         align256(static_cast<size_t>(BH) * 8 * sizeof(float));
}

// Launch that may overlap the tail of the previous kernel on the stream
// (programmatic dependent launch); the kernel waits for it with
// griddepcontrol.wait before touching that kernel's outputs.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) == cudaSuccess ? TQ_OK : TQ_ECUDA;
}

template <int BITS, int G, bool NSN>
int launch_split(const DecodeParams& p, int BH, cudaStream_t s) {
  constexpr int CB = BITS * kD / 8, SB = kD / 8;
  constexpr int STAGE = 2 * kTile * (CB + SB + 8 + (NSN ? 4 : 0));
  const size_t stage_bytes = static_cast<size_t>(kWarps) * kStages * STAGE;
  const size_t merge_bytes = static_cast<size_t>(kWarps) * G * partial_rec<NSN>() * sizeof(float);
  const size_t smem = stage_bytes > merge_bytes ? stage_bytes : merge_bytes;
  auto kern = decode_split_kernel<BITS, G, NSN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return TQ_ECUDA;
  dim3 grid(p.n_splits, BH);
  return launch_pdl(kern, grid, dim3(kWarps * 32), smem, s, p);
}

// The decode step's new rows, for the fused append (decode_prep_kernel).
struct AppendIn {
  const void* k_new;   // [B Hkv][kD] in the query's dtype, row b * Hkv + kv
  const void* v_new;
  const tq_rotation* hv;
  uint8_t* k_codes;
  uint8_t* k_signs;
  float* k_norms;
  uint8_t* v_codes;
  uint8_t* v_signs;
  float* v_norms;
  int64_t cache_stride;
  int64_t T;
  const int32_t* seq_lens;
  float* k_s1;        // NSN records (all four set, or all null): s1 of the new tokens go here,
  float* v_s1;        // and the new rows are shifted by their sequence's o before encoding
  const float* k_o;
  const float* v_o;
};

EncodeParams append_params(const tq_rotation* h, const void* x, int BH, int rope, uint8_t* codes, uint8_t* signs,
                           float* norms, float* s1) {
  EncodeParams p{};
  p.x = x;
  p.n = BH;
  p.ld = kD;
  p.pos_period = 1;
  p.rope = rope;
  p.codes = reinterpret_cast<uint32_t*>(codes);
  p.signs = reinterpret_cast<uint32_t*>(signs);
  p.norms = reinterpret_cast<float2*>(norms);
  p.out_stride = 1;
  p.nsn_s1 = s1;
  fill_handle_fields(p, h);
  return p;
}

template <typename T, int BITS>
int qprep_g(int G, int BH, const QPrepArgs<T>& a, const AppendIn* app, const tq_rotation* hk, cudaStream_t s) {
  if (!app) {
#define TQ_QPREP(GG) return launch_pdl(decode_qprep_kernel<T, GG, BITS>, dim3(BH), dim3(kD * GG), 0, s, a)
    switch (G) {
      case 1: TQ_QPREP(1);
      case 2: TQ_QPREP(2);
      case 4: TQ_QPREP(4);
      case 8: TQ_QPREP(8);
    }
#undef TQ_QPREP
    return TQ_EUNSUPPORTED;
  }
  const EncodeParams pk =
      append_params(hk, app->k_new, BH, a.rope, app->k_codes, app->k_signs, app->k_norms, app->k_s1);
  const EncodeParams pv =
      append_params(app->hv, app->v_new, BH, 0, app->v_codes, app->v_signs, app->v_norms, app->v_s1);
  const AppendArgs ap{BH, app->T, app->seq_lens, app->cache_stride, app->k_o, app->v_o};
  const unsigned blocks = static_cast<unsigned>(BH + (2 * BH + G - 1) / G);
#define TQ_PREP(GG) return launch_pdl(decode_prep_kernel<T, GG, BITS>, dim3(blocks), dim3(kD * GG), 0, s, a, ap, pk, pv)
  switch (G) {
    case 1: TQ_PREP(1);
    case 2: TQ_PREP(2);
    case 4: TQ_PREP(4);
    case 8: TQ_PREP(8);
  }
#undef TQ_PREP
  return TQ_EUNSUPPORTED;
}

template <typename T>
int qprep_b(int G, int BH, int Hkv, const T* q, const int64_t* q_pos, const tq_rotation* hk, int rope,
            uint32_t* qfrag, float4* kconst, const AppendIn* app, const float* o_k, float* qo, cudaStream_t s) {
  QPrepArgs<T> a{};
  a.o_k = o_k;
  a.qo = qo;
  a.q = q;
  a.q_pos = q_pos;
  a.Hkv = Hkv;
  a.dsigns = hk->d_signs;
  a.st = hk->d_st;
  a.rope_hi = hk->d_rope_hi;
  a.rope_lo = hk->d_rope_lo;
  a.rope_max_pos = hk->rope_max_pos;
  a.rope = rope;
  for (int i = 0; i < 4; ++i) a.walsh.w[i] = static_cast<float>(hk->walsh[i]);
  a.qfrag = qfrag;
  a.kconst = kconst;
  switch (hk->bits) {
    case 1: return qprep_g<T, 1>(G, BH, a, app, hk, s);
    case 2: return qprep_g<T, 2>(G, BH, a, app, hk, s);
    case 3: return qprep_g<T, 3>(G, BH, a, app, hk, s);
  }
  return TQ_EUNSUPPORTED;
}

int launch_qprep(int G, int q_dtype, int BH, int Hkv, const void* q, const int64_t* q_pos, const tq_rotation* hk, int rope,
                 uint32_t* qfrag, float4* kconst, const AppendIn* app, const float* o_k, float* qo, cudaStream_t s) {
  if (q_dtype == TQ_F32)
    return qprep_b<float>(G, BH, Hkv, static_cast<const float*>(q), q_pos, hk, rope, qfrag, kconst, app, o_k, qo, s);
  return qprep_b<__nv_bfloat16>(G, BH, Hkv, static_cast<const __nv_bfloat16*>(q), q_pos, hk, rope, qfrag, kconst,
                                app, o_k, qo, s);
}

// Lets `kern` take `bytes` of dynamic shared memory: past the default 48 KB
// (with its static arrays) the kernel must opt in; TQ_EUNSUPPORTED beyond
// the device's per-block maximum.
template <typename K>
int allow_dyn_smem(K kern, size_t bytes) {
  if (bytes <= 4096) return TQ_OK;   // inside the default limit for every merge instance
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return TQ_ECUDA;
  if (bytes <= static_cast<size_t>(fa.maxDynamicSharedSizeBytes)) return TQ_OK;
  int dev = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (fa.sharedSizeBytes + bytes > static_cast<size_t>(optin)) return TQ_EUNSUPPORTED;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) ==
                 cudaSuccess
             ? TQ_OK
             : TQ_ECUDA;
}

// Merge of n_parts partial records per head (layout: see decode_merge_kernel).
// final_out: the attention output [BH G][kD]; otherwise the combined partial
// records [BH G][2 + 2 kD].
int launch_merge(int G, int BH, const float* partial, int n_parts, int64_t bh_stride, int64_t part_stride,
                 const tq_rotation* hv, float* out, bool final_out, cudaStream_t s, const float* v_o = nullptr) {
  const float qjl = static_cast<float>(hv->res_const);
  // weights of the parts, [n_parts][G] floats: 37 KB at G = 8 with the most
  // splits a single sequence gets (1184)
  const size_t fsb = static_cast<size_t>(n_parts) * G * sizeof(float);
  const float* no_o = nullptr;
#define TQ_MERGE_ONE(GG, FIN, NSN, VO)                                                                         \
  {                                                                                                            \
    const int st = allow_dyn_smem(decode_merge_kernel<GG, FIN, NSN>, fsb);                                    \
    if (st != TQ_OK) return st;                                                                                \
    return launch_pdl(decode_merge_kernel<GG, FIN, NSN>, dim3(BH), dim3(kD * GG), fsb, s, partial, n_parts,   \
                      bh_stride, part_stride, hv->d_s, hv->d_signs, qjl, out, VO);                             \
  }
#define TQ_MERGE(GG)                                         \
  if (v_o) TQ_MERGE_ONE(GG, true, true, v_o)                 \
  else if (final_out) TQ_MERGE_ONE(GG, true, false, no_o)    \
  else TQ_MERGE_ONE(GG, false, false, no_o)
  switch (G) {
    case 1: TQ_MERGE(1);
    case 2: TQ_MERGE(2);
    case 4: TQ_MERGE(4);
    case 8: TQ_MERGE(8);
    default: return TQ_EUNSUPPORTED;
  }
#undef TQ_MERGE
#undef TQ_MERGE_ONE
}

template <int BITS, bool NSN>
int dispatch_g(int G, const DecodeParams& p, int BH, cudaStream_t s) {
  switch (G) {
    case 1: return launch_split<BITS, 1, NSN>(p, BH, s);
    case 2: return launch_split<BITS, 2, NSN>(p, BH, s);
    case 4: return launch_split<BITS, 4, NSN>(p, BH, s);
    case 8: return launch_split<BITS, 8, NSN>(p, BH, s);
  }
  return TQ_EUNSUPPORTED;
}

}  // namespace

extern "C" int tq_profile_next_decode(void* ev_begin, void* ev_end) {
  if ((ev_begin == nullptr) != (ev_end == nullptr)) return TQ_EINVAL;
  g_prof_begin = static_cast<cudaEvent_t>(ev_begin);
  g_prof_end = static_cast<cudaEvent_t>(ev_end);
  return TQ_OK;
}

namespace {

int launch_window(int G, int win_dtype, int q_dtype, int BH, int Hkv, const void* q, const int64_t* q_pos,
                  const tq_rotation* hk, const tq_rotation* hv, int rope, const void* k_win, const void* v_win,
                  int64_t win_stride, int R, int64_t T, const int32_t* seq_lens, float score_scale, float* partial,
                  int n_slots, int slot, cudaStream_t s) {
  const int q_f32 = q_dtype == TQ_F32 ? 1 : 0;
  const dim3 grid((R + kWinChunk - 1) / kWinChunk, BH);
#define TQ_WINDOW(TW, GG)                                                                                            \
  return launch_pdl(decode_window_kernel<TW, GG>, grid, dim3(kD), 0, s, q, q_f32, q_pos, Hkv,                         \
                    static_cast<const TW*>(k_win), static_cast<const TW*>(v_win), win_stride, R, T, seq_lens,      \
                    hv->d_signs,                                                                                   \
                    hk->d_rope_hi, hk->d_rope_lo, hk->rope_max_pos, rope, score_scale, partial, n_slots, slot)
  if (win_dtype == TQ_F32) {
    switch (G) {
      case 1: TQ_WINDOW(float, 1);
      case 2: TQ_WINDOW(float, 2);
      case 4: TQ_WINDOW(float, 4);
      case 8: TQ_WINDOW(float, 8);
    }
  } else {
    switch (G) {
      case 1: TQ_WINDOW(__nv_bfloat16, 1);
      case 2: TQ_WINDOW(__nv_bfloat16, 2);
      case 4: TQ_WINDOW(__nv_bfloat16, 4);
      case 8: TQ_WINDOW(__nv_bfloat16, 8);
    }
  }
#undef TQ_WINDOW
  return TQ_EUNSUPPORTED;
}

// One decode step over the packed cache and, when R > 0, a full-precision
// window of the R tokens after it.  Launch order: q-prep, window, split,
// merge; each waits (griddepcontrol.wait) for the launch before it, so the
// chain orders all four.
int decode_impl(const tq_rotation* hk, const tq_rotation* hv, const void* q, int q_dtype, const int64_t* q_pos,
                const uint8_t* k_codes, const uint8_t* k_signs, const float* k_norms, const uint8_t* v_codes,
                const uint8_t* v_signs, const float* v_norms, int64_t cache_stride, const void* k_win,
                const void* v_win, int win_dtype, int64_t win_stride, int R, int B, int Hq, int Hkv, int64_t T,
                const int32_t* seq_lens, float scale, float* out, float* partial_out, void* workspace,
                size_t workspace_bytes, cudaStream_t s,
                cudaEvent_t prof_begin, cudaEvent_t prof_end, const AppendIn* app = nullptr,
                const float* k_s1 = nullptr, const float* k_o = nullptr, const float* v_s1 = nullptr,
                const float* v_o = nullptr) {
  {
    const int st = check_decode_sizes(hk, hv, B, Hq, Hkv, T);
    if (st != TQ_OK) return st;
  }
  if (!q || (!out && !partial_out)) return TQ_EINVAL;
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_EINVAL;
  if (!std::isfinite(scale)) return TQ_EINVAL;
  const int G = Hq / Hkv;
  if (T > 0) {
    if (!k_codes || !k_signs || !k_norms || !v_codes || !v_signs || !v_norms) return TQ_EINVAL;
    if (cache_stride < T || (cache_stride & 1)) return TQ_EINVAL;
    const void* ptrs[6] = {k_codes, k_signs, k_norms, v_codes, v_signs, v_norms};
    for (const void* ptr : ptrs)
      if (!tq::aligned16(ptr)) return TQ_EINVAL;
  }
  const int rope = hk->rope_base > 0.0 ? 1 : 0;
  if (R < 0) return TQ_EINVAL;
  if (R > kWindowMax) return TQ_EUNSUPPORTED;
  if (R > 0) {
    if (!k_win || !v_win || win_stride < R) return TQ_EINVAL;
    if (win_dtype != TQ_F32 && win_dtype != TQ_BF16) return TQ_EINVAL;
    if (!tq::aligned16(k_win) || !tq::aligned16(v_win)) return TQ_EINVAL;   // rows are read as vectors
    if (rope && T + R > hk->rope_max_pos) return TQ_EINVAL;
  }
  if (rope && !q_pos) return TQ_EINVAL;
  const int BH = B * Hkv;
  const size_t need = workspace_for(B, Hq, Hkv, T, R);
  if (!workspace || workspace_bytes < need) return TQ_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TQ_EINVAL;
  if (!tq::on_handle_device(hk) || !tq::on_handle_device(hv)) return TQ_EINVAL;

  const SplitPlan sp = plan_splits(BH, T);
  const int n_slots = sp.n_splits + (R + kWinChunk - 1) / kWinChunk;   // window chunks after the splits
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* qfrag = reinterpret_cast<uint32_t*>(ws);
  float4* kconst = reinterpret_cast<float4*>(ws + align256(frag_bytes(BH, G)));
  float* partial = reinterpret_cast<float*>(ws + align256(frag_bytes(BH, G)) + align256(kconst_bytes(BH)));
  // NSN record mode: all four side arrays, decode over the packed cache only
  const bool nsn = k_s1 != nullptr;
  if (nsn && (!k_o || !v_s1 || !v_o || R > 0 || partial_out)) return TQ_EINVAL;
  if (app && (app->k_s1 != (nsn ? k_s1 : nullptr) || app->v_s1 != (nsn ? v_s1 : nullptr) ||
              app->k_o != (nsn ? k_o : nullptr) || app->v_o != (nsn ? v_o : nullptr)))
    return TQ_EINVAL;   // the appended records take the same side arrays as the decode
  float* qo = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(partial) +
                                       align256(static_cast<size_t>(BH) * n_slots * G * partial_rec<true>() *
                                                sizeof(float)));
  const float score_scale = scale * 1.4426950408889634f;

  int st = launch_qprep(G, q_dtype, BH, Hkv, q, q_pos, hk, rope, qfrag, kconst, app, nsn ? k_o : nullptr,
                        nsn ? qo : nullptr, s);
  if (st != TQ_OK) return st;
  st = tq::launch_status();
  if (st != TQ_OK) return st;
  if (R > 0) {
    st = launch_window(G, win_dtype, q_dtype, BH, Hkv, q, q_pos, hk, hv, rope, k_win, v_win, win_stride, R, T, seq_lens,
                       score_scale,
                       partial, n_slots, sp.n_splits, s);
    if (st != TQ_OK) return st;
  }

  DecodeParams p{};
  p.k_codes = k_codes;
  p.k_signs = k_signs;
  p.k_norms = reinterpret_cast<const float2*>(k_norms);
  p.v_codes = v_codes;
  p.v_signs = v_signs;
  p.v_norms = reinterpret_cast<const float2*>(v_norms);
  p.cache_stride = cache_stride;
  p.T = T;
  p.seq_lens = seq_lens;
  p.Hkv = Hkv;
  p.chunk = sp.chunk;
  p.n_splits = sp.n_splits;
  p.n_slots = n_slots;
  p.qfrag = qfrag;
  p.kconst = kconst;
  p.partial = partial;
  p.score_scale = score_scale;
  p.one_h = kOneH2;
  p.one_b = kOneB2;
  p.qjl = static_cast<float>(hk->res_const);
  p.append = app ? 1 : 0;
  p.k_s1 = k_s1;
  p.v_s1 = v_s1;
  p.qo = qo;
  for (int i = 0; i < 4; ++i) {
    p.walsh_k[i] = static_cast<float>(hk->walsh[i]);
    p.walsh_v[i] = static_cast<float>(hv->walsh[i]);
  }
  if (prof_begin && cudaEventRecord(prof_begin, s) != cudaSuccess) return TQ_ECUDA;
  switch (hk->bits) {
    case 1: st = nsn ? dispatch_g<1, true>(G, p, BH, s) : dispatch_g<1, false>(G, p, BH, s); break;
    case 2: st = nsn ? dispatch_g<2, true>(G, p, BH, s) : dispatch_g<2, false>(G, p, BH, s); break;
    case 3: st = nsn ? dispatch_g<3, true>(G, p, BH, s) : dispatch_g<3, false>(G, p, BH, s); break;
    default: st = TQ_EUNSUPPORTED;
  }
  if (st != TQ_OK) return st;
  if (prof_end && cudaEventRecord(prof_end, s) != cudaSuccess) return TQ_ECUDA;
  const int64_t rec = nsn ? partial_rec<true>() : partial_rec<false>();
  return launch_merge(G, BH, partial, n_slots, static_cast<int64_t>(n_slots) * G * rec, G * rec, hv,
                      partial_out ? partial_out : out, partial_out == nullptr, s, nsn ? v_o : nullptr);
}

}  // namespace

extern "C" size_t tq_decode_workspace_size(const tq_rotation* hk, const tq_rotation* hv, int B, int Hq, int Hkv,
                                           int64_t T) {
  if (check_decode_sizes(hk, hv, B, Hq, Hkv, T) != TQ_OK) return 0;
  return workspace_for(B, Hq, Hkv, T);
}

extern "C" size_t tq_decode_window_workspace_size(const tq_rotation* hk, const tq_rotation* hv, int B, int Hq,
                                                  int Hkv, int64_t T, int R) {
  if (check_decode_sizes(hk, hv, B, Hq, Hkv, T) != TQ_OK || R < 0 || R > kWindowMax) return 0;
  return workspace_for(B, Hq, Hkv, T, R);
}

extern "C" int tq_decode_attention(const tq_rotation* hk, const tq_rotation* hv, const void* q, int q_dtype,
                                   const int64_t* q_pos, const uint8_t* k_codes, const uint8_t* k_signs,
                                   const float* k_norms, const uint8_t* v_codes, const uint8_t* v_signs,
                                   const float* v_norms, int64_t cache_stride, int B, int Hq, int Hkv, int64_t T,
                                   const int32_t* seq_lens, float scale, float* out, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  const cudaEvent_t prof_begin = g_prof_begin, prof_end = g_prof_end;
  g_prof_begin = g_prof_end = nullptr;
  return decode_impl(hk, hv, q, q_dtype, q_pos, k_codes, k_signs, k_norms, v_codes, v_signs, v_norms, cache_stride,
                     nullptr, nullptr, TQ_F32, 0, 0, B, Hq, Hkv, T, seq_lens, scale, out, nullptr, workspace,
                     workspace_bytes,
                     static_cast<cudaStream_t>(stream), prof_begin, prof_end);
}

extern "C" int tq_decode_attention_append(const tq_rotation* hk, const tq_rotation* hv, const void* q, int q_dtype,
                                          const int64_t* q_pos, const void* k_new, const void* v_new,
                                          uint8_t* k_codes, uint8_t* k_signs, float* k_norms, uint8_t* v_codes,
                                          uint8_t* v_signs, float* v_norms, int64_t cache_stride, int B, int Hq,
                                          int Hkv, int64_t T, const int32_t* seq_lens, float scale, float* out,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!k_new || !v_new) return TQ_EINVAL;
  const cudaEvent_t prof_begin = g_prof_begin, prof_end = g_prof_end;
  g_prof_begin = g_prof_end = nullptr;
  AppendIn app{k_new, v_new, hv, k_codes, k_signs, k_norms, v_codes, v_signs, v_norms, cache_stride, T, seq_lens};
  return decode_impl(hk, hv, q, q_dtype, q_pos, k_codes, k_signs, k_norms, v_codes, v_signs, v_norms, cache_stride,
                     nullptr, nullptr, TQ_F32, 0, 0, B, Hq, Hkv, T, seq_lens, scale, out, nullptr, workspace,
                     workspace_bytes, static_cast<cudaStream_t>(stream), prof_begin, prof_end, &app);
}

extern "C" int tq_decode_attention_nsn(const tq_rotation* hk, const tq_rotation* hv, const void* q, int q_dtype,
                                       const int64_t* q_pos, const uint8_t* k_codes, const uint8_t* k_signs,
                                       const float* k_norms, const uint8_t* v_codes, const uint8_t* v_signs,
                                       const float* v_norms, const float* k_s1, const float* k_o, const float* v_s1,
                                       const float* v_o, int64_t cache_stride, int B, int Hq, int Hkv, int64_t T,
                                       const int32_t* seq_lens, float scale, float* out, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (!k_s1 || !k_o || !v_s1 || !v_o) return TQ_EINVAL;
  if (T > 0 && (!tq::aligned16(k_s1) || !tq::aligned16(v_s1))) return TQ_EINVAL;   // copied 16 bytes at a time
  if (cache_stride % 4) return TQ_EINVAL;   // each sequence's s1 row starts 16-byte aligned
  const cudaEvent_t prof_begin = g_prof_begin, prof_end = g_prof_end;
  g_prof_begin = g_prof_end = nullptr;
  return decode_impl(hk, hv, q, q_dtype, q_pos, k_codes, k_signs, k_norms, v_codes, v_signs, v_norms, cache_stride,
                     nullptr, nullptr, TQ_F32, 0, 0, B, Hq, Hkv, T, seq_lens, scale, out, nullptr, workspace,
                     workspace_bytes, static_cast<cudaStream_t>(stream), prof_begin, prof_end, nullptr, k_s1, k_o,
                     v_s1, v_o);
}

extern "C" int tq_decode_attention_nsn_append(const tq_rotation* hk, const tq_rotation* hv, const void* q,
                                              int q_dtype, const int64_t* q_pos, const void* k_new,
                                              const void* v_new, uint8_t* k_codes, uint8_t* k_signs, float* k_norms,
                                              uint8_t* v_codes, uint8_t* v_signs, float* v_norms, float* k_s1,
                                              const float* k_o, float* v_s1, const float* v_o,
                                              int64_t cache_stride, int B, int Hq, int Hkv, int64_t T,
                                              const int32_t* seq_lens, float scale, float* out, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  if (!k_new || !v_new || !k_s1 || !k_o || !v_s1 || !v_o) return TQ_EINVAL;
  if (T > 0 && (!tq::aligned16(k_s1) || !tq::aligned16(v_s1))) return TQ_EINVAL;   // copied 16 bytes at a time
  if (cache_stride % 4) return TQ_EINVAL;   // each sequence's s1 row starts 16-byte aligned
  const cudaEvent_t prof_begin = g_prof_begin, prof_end = g_prof_end;
  g_prof_begin = g_prof_end = nullptr;
  AppendIn app{k_new, v_new, hv, k_codes, k_signs, k_norms, v_codes, v_signs, v_norms, cache_stride, T, seq_lens,
               k_s1, v_s1, k_o, v_o};
  return decode_impl(hk, hv, q, q_dtype, q_pos, k_codes, k_signs, k_norms, v_codes, v_signs, v_norms, cache_stride,
                     nullptr, nullptr, TQ_F32, 0, 0, B, Hq, Hkv, T, seq_lens, scale, out, nullptr, workspace,
                     workspace_bytes, static_cast<cudaStream_t>(stream), prof_begin, prof_end, &app, k_s1, k_o, v_s1,
                     v_o);
}

extern "C" int tq_decode_attention_window(const tq_rotation* hk, const tq_rotation* hv, const void* q, int q_dtype,
                                          const int64_t* q_pos, const uint8_t* k_codes, const uint8_t* k_signs,
                                          const float* k_norms, const uint8_t* v_codes, const uint8_t* v_signs,
                                          const float* v_norms, int64_t cache_stride, const void* k_window,
                                          const void* v_window, int window_dtype, int64_t window_stride, int R,
                                          int B, int Hq, int Hkv, int64_t T, const int32_t* seq_lens, float scale,
                                          float* out, void* workspace, size_t workspace_bytes, void* stream) {
  const cudaEvent_t prof_begin = g_prof_begin, prof_end = g_prof_end;
  g_prof_begin = g_prof_end = nullptr;
  return decode_impl(hk, hv, q, q_dtype, q_pos, k_codes, k_signs, k_norms, v_codes, v_signs, v_norms, cache_stride,
                     k_window, v_window, window_dtype, window_stride, R, B, Hq, Hkv, T, seq_lens, scale, out, nullptr,
                     workspace, workspace_bytes, static_cast<cudaStream_t>(stream), prof_begin, prof_end);
}

extern "C" int tq_decode_partials(const tq_rotation* hk, const tq_rotation* hv, const void* q, int q_dtype,
                                  const int64_t* q_pos, const uint8_t* k_codes, const uint8_t* k_signs,
                                  const float* k_norms, const uint8_t* v_codes, const uint8_t* v_signs,
                                  const float* v_norms, int64_t cache_stride, int B, int Hq, int Hkv, int64_t T,
                                  const int32_t* seq_lens, float scale, float* partials, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (!partials) return TQ_EINVAL;
  return decode_impl(hk, hv, q, q_dtype, q_pos, k_codes, k_signs, k_norms, v_codes, v_signs, v_norms, cache_stride,
                     nullptr, nullptr, TQ_F32, 0, 0, B, Hq, Hkv, T, seq_lens, scale, nullptr, partials, workspace,
                     workspace_bytes, static_cast<cudaStream_t>(stream), nullptr, nullptr);
}

extern "C" int tq_decode_merge_partials(const tq_rotation* hv, const float* partials, int n_parts, int B, int Hq,
                                        int Hkv, float* out, void* stream) {
  if (!hv || !partials || !out || n_parts < 1 || n_parts > (1 << 16)) return TQ_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv) return TQ_EINVAL;
  if (static_cast<int64_t>(B) * Hkv > kMaxSequences) return TQ_EUNSUPPORTED;
  if (hv->d != kD || hv->m != kD || hv->kind != TQ_ROT_HADAMARD) return TQ_EUNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return TQ_EUNSUPPORTED;
  if (!tq::on_handle_device(hv)) return TQ_EINVAL;
  const int BH = B * Hkv;
  const int64_t rec = 2 + 2 * kD;
  const int st = launch_merge(G, BH, partials, n_parts, G * rec, static_cast<int64_t>(BH) * G * rec, hv, out, true,
                              static_cast<cudaStream_t>(stream));
  return st != TQ_OK ? st : tq::launch_status();
}

// ---------------------------------------------------------------------------
// Decode attention without any allocation (tq_decode_attention_noalloc).
//
// Some callers cannot call cudaMalloc: runtimes that own the device memory
// budget and forbid allocation once serving starts, hosts that hand the
// library no allocator, or paths that must never block on or fail in an
// allocation.  For them the scratch of tq_decode_attention (query operand
// fragments, per-head constants, split partials) lives in the fixed array
// below, which every device that loads this library holds until exit.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB per device
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_scratch_addr[kNoAllocMaxDevices] = {};
}  // namespace

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

extern "C" int tq_decode_attention_noalloc(const tq_rotation* hk, const tq_rotation* hv, const void* q, int q_dtype,
                                           const int64_t* q_pos, const uint8_t* k_codes, const uint8_t* k_signs,
                                           const float* k_norms, const uint8_t* v_codes, const uint8_t* v_signs,
                                           const float* v_norms, int64_t cache_stride, int B, int Hq, int Hkv,
                                           int64_t T, const int32_t* seq_lens, float scale, float* out,
                                           void* stream) {
  // the handle and size checks of tq_decode_attention come first, so a call
  // this library cannot serve at all reports that rather than the cap below
  {
    const int st = check_decode_sizes(hk, hv, B, Hq, Hkv, T);
    if (st != TQ_OK) return st;
  }
  if (workspace_for(B, Hq, Hkv, T) > kNoAllocScratchBytes) return TQ_EWORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return TQ_ECUDA;
  void* scratch = nullptr;
  {
    // First call on a device: look up this device's copy of the array.  The
    // host-side name of a __device__ variable is only a stand-in, never a
    // device address, so the address must come from the runtime.
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_scratch_addr[dev]) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) {
        cudaGetLastError();
        return TQ_ECUDA;
      }
      g_noalloc_scratch_addr[dev] = addr;
    }
    scratch = g_noalloc_scratch_addr[dev];
  }
  return tq_decode_attention(hk, hv, q, q_dtype, q_pos, k_codes, k_signs, k_norms, v_codes, v_signs, v_norms,
                             cache_stride, B, Hq, Hkv, T, seq_lens, scale, out, scratch, kNoAllocScratchBytes,
                             stream);
}
