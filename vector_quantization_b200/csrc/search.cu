// Brute-force inner-product top-k search over packed vectors.
//
// [TurboQuant] "Expériences et résultats" / "Performances en recherche
// vectorielle": the codec serves maximum-inner-product search without large
// codebooks.  Each database vector x_n is scored by the same estimator as
// attention,
//   score(q, n) = ||x_n|| <Pi q, c[idx_n]> + ||r_n|| sqrt(pi/2)/m <S Pi q, sign(S r_n)>,
// and the k best per query are kept (ties to the lower id).
//
// Launches: q-prep (q~ = Pi q and s = S q~ as fp32 GEMMs for a dense
// rotation), a fragment kernel (fp16 operands of q~ and s, scaled into fp16
// range per query, divided by the per-slot sigma of the bit operand), the
// scoring kernel, and a merge of the per-range candidate lists.
//
// Scoring kernel: one CTA = 16 queries x a range of database rows.  The
// queries' B fragments (all d dims) stay resident in shared memory; 8 warps
// take 16 database rows each per 128-row tile and build the A operand of
// mma.sync m16n8k16 (fp16, fp32 accumulate) straight from the packed code and
// sign bit-planes with one LOP3 per register (bitplane.cuh).  Code planes are
// in Walsh form, so they are exact; the query side is a single fp16 piece
// (2^-12 relative), well inside the score tolerance for this workload.  Each
// warp keeps the running top-k of 2 queries in registers (lane i = rank i),
// inserting candidates warp-parallel.
#include <cmath>

#include "bitplane.cuh"
#include "tq_internal.h"

namespace tq {
int sgemm_nt(int M, int N, int K, const float* A, int64_t lda, const float* B, int64_t ldb, float* C, int64_t ldc,
             cudaStream_t s);
}

namespace {

using namespace tqdev;

constexpr int kQT = 16;          // queries per CTA
constexpr int kRowsPerWarp = 16;
constexpr int kSWarps = 8;
constexpr int kTileRows = kSWarps * kRowsPerWarp;   // 128 database rows per tile
constexpr int kQPW = kQT / kSWarps;                 // queries whose top-k one warp keeps
constexpr int kMaxK = 32;

struct SearchParams {
  const uint8_t* codes;
  const uint8_t* signs;
  const float2* norms;
  int64_t N;
  int64_t range;              // database rows per CTA range (multiple of kTileRows)
  int nq, k, d, nblk;         // nblk = d / 128
  const uint32_t* qfrag;      // [qtile][nblk][2][8][2][32][2]
  const float4* qconst;       // [nq_pad]: (K_q, 1/lam_q, K_s, 1/lam_s)
  float qjl;
  float walsh[4];
  uint32_t one_h;             // kOneH2, passed at run time (see bit_select)
  float* cand_score;          // [n_ranges][nq][k]
  int64_t* cand_id;
};

__device__ __forceinline__ bool better(float s1, int64_t i1, float s2, int64_t i2) {
  return s1 > s2 || (s1 == s2 && i1 < i2);
}

// Warp-parallel insertion into a sorted list held one entry per lane.
__device__ __forceinline__ void topk_insert(float& ls, int64_t& li, int lane, int k, float s, int64_t id) {
  const bool ahead = lane < k && better(ls, li, s, id);
  const int pos = __popc(__ballot_sync(0xffffffffu, ahead));
  if (pos >= k) return;
  const float ps = __shfl_up_sync(0xffffffffu, ls, 1);
  const int64_t pi = __shfl_up_sync(0xffffffffu, li, 1);
  if (lane > pos && lane < k) {
    ls = ps;
    li = pi;
  }
  if (lane == pos) {
    ls = s;
    li = id;
  }
}

template <int BITS>
__global__ void __launch_bounds__(kSWarps * 32) search_score_kernel(SearchParams p) {
  constexpr int P = Planes<BITS>::P;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* bfr = reinterpret_cast<uint32_t*>(smem);                                 // query fragments
  float* sc = reinterpret_cast<float*>(smem + static_cast<size_t>(p.nblk) * 2 * 8 * 2 * 32 * 2 * 4);  // [kQT][64]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int qtile = blockIdx.x;
  const int range = blockIdx.y;
  const int64_t r_begin = static_cast<int64_t>(range) * p.range;
  const int64_t r_end = min(p.N, r_begin + p.range);
  const int cb = BITS * p.d / 8, sb = p.d / 8;

  {
    const int words = p.nblk * 2 * 8 * 2 * 32 * 2;
    const uint32_t* src = p.qfrag + static_cast<size_t>(qtile) * words;
    for (int i = threadIdx.x * 4; i < words; i += blockDim.x * 4) cp_async16(bfr + i, src + i, 16);
    cp_async_commit();
  }
  float4 qc[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) qc[nt][e] = p.qconst[qtile * kQT + 8 * nt + 2 * tig + e];
  // this warp's running top-k of queries kQPW warp .. (lane = rank)
  float ls[kQPW];
  int64_t li[kQPW];
#pragma unroll
  for (int j = 0; j < kQPW; ++j) {
    ls[j] = -INFINITY;
    li[j] = INT64_MAX;
  }
  cp_async_wait<0>();
  __syncthreads();

  for (int64_t t0 = r_begin; t0 < r_end; t0 += kTileRows) {
    const int64_t row0 = t0 + warp * kRowsPerWarp + gid, row1 = row0 + 8;
    const bool v0 = row0 < r_end, v1 = row1 < r_end;
    const uint8_t* c0 = p.codes + (v0 ? row0 : r_begin) * cb;
    const uint8_t* c1 = p.codes + (v1 ? row1 : r_begin) * cb;
    const uint8_t* s0p = p.signs + (v0 ? row0 : r_begin) * sb;
    const uint8_t* s1p = p.signs + (v1 ? row1 : r_begin) * sb;
    float cacc[P][2][4], zacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int r = 0; r < 4; ++r) zacc[nt][r] = 0.f;
#pragma unroll
      for (int pl = 0; pl < P; ++pl)
#pragma unroll
        for (int r = 0; r < 4; ++r) cacc[pl][nt][r] = 0.f;
    }
    // word tig of 128-dim block blk of every plane (and of the signs), rows
    // gid and gid + 8; the next block's words are loaded one block ahead
    uint32_t nx0[BITS + 1], nx1[BITS + 1];
    auto load_words = [&](int blk) {
#pragma unroll
      for (int k = 0; k < BITS; ++k) {
        nx0[k] = __ldg(reinterpret_cast<const uint32_t*>(c0 + k * (p.d / 8)) + 4 * blk + tig);
        nx1[k] = __ldg(reinterpret_cast<const uint32_t*>(c1 + k * (p.d / 8)) + 4 * blk + tig);
      }
      nx0[BITS] = __ldg(reinterpret_cast<const uint32_t*>(s0p) + 4 * blk + tig);
      nx1[BITS] = __ldg(reinterpret_cast<const uint32_t*>(s1p) + 4 * blk + tig);
    };
    load_words(0);
#pragma unroll 1
    for (int blk = 0; blk < p.nblk; ++blk) {
      uint32_t raw0[BITS], raw1[BITS];
#pragma unroll
      for (int k = 0; k < BITS; ++k) {
        raw0[k] = nx0[k];
        raw1[k] = nx1[k];
      }
      uint32_t w0[P + 1], w1[P + 1];
      {
        uint32_t pl0[P], pl1[P];
        Planes<BITS>::make(raw0, pl0);
        Planes<BITS>::make(raw1, pl1);
#pragma unroll
        for (int q = 0; q < P; ++q) {
          w0[q] = pl0[q];
          w1[q] = pl1[q];
        }
        w0[P] = nx0[BITS];
        w1[P] = nx1[BITS];
      }
      if (blk + 1 < p.nblk) load_words(blk + 1);
      uint32_t ws0[P + 1], ws1[P + 1];
#pragma unroll
      for (int q = 0; q <= P; ++q) {
        ws0[q] = w0[q] << 8;
        ws1[q] = w1[q] << 8;
      }
      const uint32_t* bb = bfr + static_cast<size_t>(blk) * (2 * 8 * 2 * 32 * 2);
#pragma unroll
      for (int kb = 0; kb < 8; ++kb) {
        uint2 bq[2][2];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
            bq[t][nt] = *reinterpret_cast<const uint2*>(bb + (((t * 8 + kb) * 2 + nt) * 32 + lane) * 2);
#pragma unroll
        for (int q = 0; q <= P; ++q) {
          const uint32_t a[4] = {bit_pair_h(w0[q], ws0[q], 2 * kb, p.one_h), bit_pair_h(w1[q], ws1[q], 2 * kb, p.one_h),
                                 bit_pair_h(w0[q], ws0[q], 2 * kb + 1, p.one_h),
                                 bit_pair_h(w1[q], ws1[q], 2 * kb + 1, p.one_h)};
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            if (q < P) mma_f16(cacc[q < P ? q : 0][nt], a, bq[0][nt].x, bq[0][nt].y);
            else mma_f16(zacc[nt], a, bq[1][nt].x, bq[1][nt].y);
          }
        }
      }
    }
    // ---- scores into shared memory [query][row in tile] ----------------------
    const float2 n0 = v0 ? p.norms[row0] : make_float2(0.f, 0.f);
    const float2 n1 = v1 ? p.norms[row1] : make_float2(0.f, 0.f);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float4 c = qc[nt][e];
        float code0 = 0.f, code1 = 0.f;
#pragma unroll
        for (int pl = 0; pl < P; ++pl) {
          code0 = fmaf(p.walsh[pl], (cacc[pl][nt][e] - c.x) * c.y, code0);
          code1 = fmaf(p.walsh[pl], (cacc[pl][nt][2 + e] - c.x) * c.y, code1);
        }
        const float z0 = (zacc[nt][e] - c.z) * c.w, z1 = (zacc[nt][2 + e] - c.z) * c.w;
        const int qq = 8 * nt + 2 * tig + e;
        sc[qq * kTileRows + warp * kRowsPerWarp + gid] = v0 ? fmaf(n0.x, code0, n0.y * p.qjl * z0) : -INFINITY;
        sc[qq * kTileRows + warp * kRowsPerWarp + gid + 8] = v1 ? fmaf(n1.x, code1, n1.y * p.qjl * z1) : -INFINITY;
      }
    __syncthreads();
    // ---- top-k update: warp w owns queries kQPW w .. kQPW w + kQPW - 1 ---------
#pragma unroll
    for (int j = 0; j < kQPW; ++j) {
      const int qq = kQPW * warp + j;
      const float thr = __shfl_sync(0xffffffffu, ls[j], p.k - 1);
      const int64_t thr_id = __shfl_sync(0xffffffffu, li[j], p.k - 1);
#pragma unroll
      for (int half = 0; half < kTileRows / 32; ++half) {
        const int rr = half * 32 + lane;
        const float s = sc[qq * kTileRows + rr];
        const int64_t id = t0 + rr;
        unsigned cand = __ballot_sync(0xffffffffu, s != -INFINITY && better(s, id, thr, thr_id));
        while (cand) {
          const int src = __ffs(cand) - 1;
          cand &= cand - 1;
          const float cs = __shfl_sync(0xffffffffu, s, src);
          topk_insert(ls[j], li[j], lane, p.k, cs, t0 + half * 32 + src);
        }
      }
    }
    __syncthreads();
  }
  // ---- write this range's candidates ---------------------------------------
#pragma unroll
  for (int j = 0; j < kQPW; ++j) {
    const int q = qtile * kQT + kQPW * warp + j;
    if (q < p.nq && lane < p.k) {
      const size_t o = (static_cast<size_t>(range) * p.nq + q) * p.k + lane;
      p.cand_score[o] = ls[j];
      p.cand_id[o] = li[j] == INT64_MAX ? -1 : li[j];
    }
  }
}

// One warp per query: merge the candidate lists of all ranges.
// One warp per query: the best k of n_ranges candidate lists [n_ranges][nq][k]
// (descending score, ties to the lower id); list r's ids are shifted by
// id_offsets[r] when id_offsets is given (lists of database shards).
__global__ void search_merge_kernel(const float* __restrict__ cs, const int64_t* __restrict__ ci, int n_ranges, int nq,
                                    int k, const int64_t* __restrict__ id_offsets, float* __restrict__ scores,
                                    int64_t* __restrict__ ids) {
  const int lane = threadIdx.x & 31;
  const int q = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (q >= nq) return;
  float ls = -INFINITY;
  int64_t li = INT64_MAX;
  for (int r = 0; r < n_ranges; ++r) {
    const size_t base = (static_cast<size_t>(r) * nq + q) * k;
    const float s = lane < k ? cs[base + lane] : -INFINITY;
    int64_t id = lane < k ? ci[base + lane] : -1;
    if (id_offsets && id >= 0) id += id_offsets[r];
    unsigned cand = __ballot_sync(0xffffffffu, id >= 0 && s != -INFINITY);
    while (cand) {
      const int src = __ffs(cand) - 1;
      cand &= cand - 1;
      topk_insert(ls, li, lane, k, __shfl_sync(0xffffffffu, s, src), __shfl_sync(0xffffffffu, id, src));
    }
  }
  if (lane < k) {
    scores[static_cast<size_t>(q) * k + lane] = ls;
    ids[static_cast<size_t>(q) * k + lane] = li == INT64_MAX ? -1 : li;
  }
}

// One block of 128 threads per query: fp16 B fragments of q~ and s.
__global__ void __launch_bounds__(128) search_frag_kernel(const float* __restrict__ qt, const float* __restrict__ sq,
                                                          int nq, int d, int nblk, uint16_t* __restrict__ qfrag,
                                                          float4* __restrict__ qconst) {
  __shared__ float red[4];
  const int q = blockIdx.x;
  const int tid = threadIdx.x;
  const int qtile = q / kQT, ql = q % kQT;
  const int gid = ql & 7, nt = ql >> 3;
  float out_c[2], out_l[2];
#pragma unroll
  for (int type = 0; type < 2; ++type) {
    const float* src = (type == 0 ? qt : sq) + static_cast<size_t>(q) * d;
    float mx = 0.f;
    for (int i = tid; i < d; i += 128) {
      const int j = i & 15;
      const int pp = slot_pos(j);
      mx = fmaxf(mx, fabsf(src[i] / (0.5f * (pos_v1_h(pp) - pos_v0_h(pp)))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();
    const float lam = fp16_range_scale(mx);
    float c = 0.f;
    for (int i = tid; i < d; i += 128) {
      const int blk = i >> 7, ii = i & 127;
      const int tg = ii >> 5, x = ii & 31, e = x >> 4, j = x & 15, reg = j & 1, kb = j >> 1;
      const int pp = slot_pos(j);
      const float mu = 0.5f * (pos_v0_h(pp) + pos_v1_h(pp)), sigma = 0.5f * (pos_v1_h(pp) - pos_v0_h(pp));
      const __half h = __float2half_rn(src[i] / sigma * lam);
      c += mu * __half2float(h);
      const int ln = 4 * gid + tg;
      const size_t idx =
          ((((((static_cast<size_t>(qtile) * nblk + blk) * 2 + type) * 8 + kb) * 2 + nt) * 32 + ln) * 2 + reg) * 2 + e;
      qfrag[idx] = __half_as_ushort(h);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if ((tid & 31) == 0) red[tid >> 5] = c;
    __syncthreads();
    out_c[type] = red[0] + red[1] + red[2] + red[3];
    out_l[type] = 1.0f / lam;
    __syncthreads();
  }
  if (tid == 0) qconst[q] = make_float4(out_c[0], out_l[0], out_c[1], out_l[1]);
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

struct SearchPlan {
  int qtiles, n_ranges;
  int64_t range;
};

SearchPlan plan(int nq, int64_t N) {
  SearchPlan sp{};
  sp.qtiles = (nq + kQT - 1) / kQT;
  // about 32 CTAs per SM in all (16 waves at two per SM), so the last wave's
  // tail is a small part of the run (2 per SM gave 29.3 ms for 1M x 1536
  // rows and 1000 queries at 1+1 bits, 16 per SM 21.9 ms, 32 per SM 21.1 ms)
  int64_t want = (32 * 148 + sp.qtiles / 2) / sp.qtiles;
  const int64_t max_ranges = (N + kTileRows - 1) / kTileRows;
  if (want > max_ranges) want = max_ranges;
  if (want < 1) want = 1;
  int64_t range = (N + want - 1) / want;
  range = (range + kTileRows - 1) / kTileRows * kTileRows;
  if (range < kTileRows) range = kTileRows;
  sp.range = range;
  sp.n_ranges = static_cast<int>((N + range - 1) / range);
  if (sp.n_ranges < 1) sp.n_ranges = 1;
  return sp;
}

struct SearchLayout {
  size_t qt, sq, frag, qconst, cs, ci, total;
};

SearchLayout layout(const tq_rotation* h, int nq, int64_t N, int k) {
  const SearchPlan sp = plan(nq, N);
  const size_t nq_pad = static_cast<size_t>(sp.qtiles) * kQT;
  SearchLayout L{};
  size_t off = 0;
  L.qt = off;
  off += align256(nq_pad * h->d * sizeof(float));
  L.sq = off;
  off += align256(nq_pad * h->m * sizeof(float));
  L.frag = off;
  off += align256(static_cast<size_t>(sp.qtiles) * (h->d / 128) * 2 * 8 * 2 * 32 * 2 * 4);
  L.qconst = off;
  off += align256(nq_pad * sizeof(float4));
  L.cs = off;
  off += align256(static_cast<size_t>(sp.n_ranges) * nq * k * sizeof(float));
  L.ci = off;
  off += align256(static_cast<size_t>(sp.n_ranges) * nq * k * sizeof(int64_t));
  L.total = off;
  return L;
}

template <int BITS>
int launch_score(const SearchParams& p, const SearchPlan& sp, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(p.nblk) * 2 * 8 * 2 * 32 * 2 * 4 + kQT * kTileRows * sizeof(float);
  auto kern = search_score_kernel<BITS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return TQ_ECUDA;
  dim3 grid(sp.qtiles, sp.n_ranges);
  kern<<<grid, kSWarps * 32, smem, s>>>(p);
  return tq::launch_status();
}

}  // namespace

extern "C" size_t tq_search_workspace_size(const tq_rotation* h, int nq, int64_t N, int k) {
  if (!h || nq < 1 || N < 0 || k < 1 || k > kMaxK) return 0;
  return layout(h, nq, N, k).total;
}

extern "C" int tq_search_topk(const tq_rotation* h, const float* queries, int nq, const uint8_t* codes,
                              const uint8_t* signs, const float* norms, int64_t N, int k, float* scores, int64_t* ids,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (!h || !queries || !scores || !ids || nq < 1 || N < 0 || k < 1 || k > kMaxK) return TQ_EINVAL;
  if (h->kind != TQ_ROT_DENSE) return TQ_EUNSUPPORTED;
  if (h->d % 128 || h->m != h->d) return TQ_EUNSUPPORTED;
  if (N > 0 && (!codes || !signs || !norms)) return TQ_EINVAL;
  if (!tq::aligned16(queries) || (N > 0 && (!tq::aligned16(codes) || !tq::aligned16(signs) || !tq::aligned16(norms))))
    return TQ_EINVAL;
  const SearchLayout L = layout(h, nq, N, k);
  if (!workspace || workspace_bytes < L.total) return TQ_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TQ_EINVAL;
  if (!tq::on_handle_device(h)) return TQ_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const SearchPlan sp = plan(nq, N);
  const int d = h->d, m = h->m;
  float* qt = reinterpret_cast<float*>(ws + L.qt);
  float* sq = reinterpret_cast<float*>(ws + L.sq);
  const int nq_pad = sp.qtiles * kQT;
  // padded query rows are zero so their fragments are finite
  if (cudaMemsetAsync(qt, 0, static_cast<size_t>(nq_pad) * d * sizeof(float), s) != cudaSuccess) return TQ_ECUDA;
  int st = tq::sgemm_nt(nq, d, d, queries, d, h->d_pi, d, qt, d, s);   // q~ = Pi q
  if (st != TQ_OK) return st;
  if ((st = tq::sgemm_nt(nq_pad, m, d, qt, d, h->d_s, d, sq, m, s)) != TQ_OK) return st;   // s = S q~
  search_frag_kernel<<<nq_pad, 128, 0, s>>>(qt, sq, nq_pad, d, d / 128, reinterpret_cast<uint16_t*>(ws + L.frag),
                                            reinterpret_cast<float4*>(ws + L.qconst));
  if ((st = tq::launch_status()) != TQ_OK) return st;
  SearchParams p{};
  p.codes = codes;
  p.signs = signs;
  p.norms = reinterpret_cast<const float2*>(norms);
  p.N = N;
  p.range = sp.range;
  p.nq = nq;
  p.k = k;
  p.d = d;
  p.nblk = d / 128;
  p.qfrag = reinterpret_cast<const uint32_t*>(ws + L.frag);
  p.qconst = reinterpret_cast<const float4*>(ws + L.qconst);
  p.qjl = static_cast<float>(h->res_const);
  for (int i = 0; i < 4; ++i) p.walsh[i] = static_cast<float>(h->walsh[i]);
  p.one_h = kOneH2;
  p.cand_score = reinterpret_cast<float*>(ws + L.cs);
  p.cand_id = reinterpret_cast<int64_t*>(ws + L.ci);
  switch (h->bits) {
    case 1: st = launch_score<1>(p, sp, s); break;
    case 2: st = launch_score<2>(p, sp, s); break;
    default: st = launch_score<3>(p, sp, s); break;
  }
  if (st != TQ_OK) return st;
  search_merge_kernel<<<(nq + 7) / 8, 256, 0, s>>>(p.cand_score, p.cand_id, sp.n_ranges, nq, k, nullptr, scores, ids);
  return tq::launch_status();
}

extern "C" int tq_search_merge_topk(const float* cand_scores, const int64_t* cand_ids, int n_lists, int nq, int k,
                                    const int64_t* id_offsets, float* scores, int64_t* ids, void* stream) {
  if (!cand_scores || !cand_ids || !scores || !ids || n_lists < 1 || nq < 1 || k < 1 || k > kMaxK) return TQ_EINVAL;
  search_merge_kernel<<<(nq + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(cand_scores, cand_ids, n_lists, nq,
                                                                                    k, id_offsets, scores, ids);
  return tq::launch_status();
}
