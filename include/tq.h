/*
 * tq.h - C ABI of the B200 rotation + Lloyd-Max + QJL vector codec.
 *
 * The codec (TurboQuant-style; sources named per entry point):
 *   encode:  RoPE (keys only) -> rotation Pi -> per-coordinate b-bit
 *            Lloyd-Max code + vector norm -> 1-bit QJL sketch sign(S r) of
 *            the residual r plus ||r||, bit-packed;
 *   decode:  attention scored straight from the packed cache, one pass.
 *
 * Conventions for every entry point:
 *   - All pointers named "device" are CUDA device pointers on the device the
 *     handle was built on; "host" pointers are ordinary host memory.
 *   - The caller owns every buffer it passes.  The library allocates device
 *     memory only inside tq_build_rotation (owned by the handle, released by
 *     tq_free_rotation).
 *   - Calls that launch kernels are asynchronous on `stream` (a cudaStream_t
 *     passed as void*; NULL = legacy default stream).  Arguments are checked
 *     on the host before anything is launched; a rejected call launches
 *     nothing and returns a negative status.  Launch failures return
 *     TQ_ECUDA; faults inside a kernel surface at the caller's next
 *     synchronisation, as with any CUDA call.
 *   - Nothing is thrown across the ABI.  Handles are immutable after build
 *     and may be shared between threads and streams.
 *
 * Packed record of one vector (bits b, dimension d, sketch size m):
 *   codes  b*d/8 bytes: b bit-planes of d bits, plane k holds bit k of every
 *          code; coordinate i at byte i/8, bit i%8; planes in order k=0..b-1.
 *          Codes number the Lloyd-Max levels in ascending order.
 *   signs  m/8 bytes: bit j = 1 iff (S r)_j >= 0, same bit order.
 *   norms  two float32: ||x|| (after RoPE) and ||r||.
 * Codes, signs and norms live in three separate arrays indexed by record.
 *
 * Sources (pages, cited by title and section):
 *   [TurboESM]   "TurboESM: Ultra-Efficient 3-Bit KV Cache Quantization for
 *                Protein Language Models with Orthogonal Rotation and QJL
 *                Correction", Résumé technique §2.A-§2.E.
 *   [TurboQuant] TurboQuant digest (news.hada.io 27867): "Principe de
 *                fonctionnement" (Étape 1, Étape 2), "QJL", "Expériences et
 *                résultats".
 *   [NSNQuant]   "NSNQuant: ...", Résumé Technique, Méthodologie §2 and
 *                §4 ("Résidus": the full-precision window).
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define TQ_OK            0
#define TQ_EINVAL       -1   /* bad argument (null pointer, size, alignment) */
#define TQ_EUNSUPPORTED -2   /* valid but not implemented (d, bits, heads)   */
#define TQ_EWORKSPACE   -3   /* workspace missing or too small               */
#define TQ_ECUDA        -4   /* a CUDA runtime call or launch failed         */
#define TQ_ENOMEM       -5   /* device allocation failed                     */

/* ---- enumerations ------------------------------------------------------ */
#define TQ_ROT_HADAMARD  0   /* Pi = H_d diag(D) / sqrt(d), d a power of two */
#define TQ_ROT_DENSE     1   /* Pi = Q diag(sign(diag R)), G = QR, any d     */

#define TQ_F32           0   /* float32 elements */
#define TQ_BF16          1   /* bfloat16 elements */

/* Residual correction of a handle ([TurboQuant] Étape 2 / [TurboESM] §2.D). */
#define TQ_RES_QJL       0   /* sign(S r) and ||r||; estimator sqrt(pi/2)/m   */
#define TQ_RES_SIGN      1   /* sign(r) and mean |r_i|; x~ = x^ + e sign(r)   */

typedef struct tq_rotation tq_rotation;

/* Human-readable text for a status code (static storage). */
const char* tq_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int tq_version(void);

/*
 * tq_lloyd_max - host only; the scalar codebook the codec uses.
 * [TurboQuant] "Principe", Étape 1 and comments: after a random rotation a
 * standard quantizer, its boundaries and levels optimised by Lloyd-Max, is
 * applied to each coordinate.  The law quantized is the exact density of one
 * coordinate of a uniform point on S^{d-1}, f(t) ~ (1-t^2)^((d-3)/2).
 *   d           dimension, 3 <= d <= 65536
 *   bits        1..8
 *   levels      host out [2^bits] ascending reconstruction levels (float64)
 *   thresholds  host out [2^bits - 1], thresholds[j] = (levels[j]+levels[j+1])/2
 * Returns TQ_OK or TQ_EINVAL.  Pure host computation; needs no GPU.
 */
int tq_lloyd_max(int d, int bits, double* levels, double* thresholds);

/*
 * tq_build_rotation - build a codec handle on the current CUDA device.
 * [TurboQuant] Étape 1 (data-oblivious random rotation), [NSNQuant] §2
 * (randomized Hadamard), [TurboQuant] "QJL" (Gaussian projection S),
 * [TurboESM] §2.A (RoPE before the rotation).
 *   d          vector dimension; TQ_ROT_HADAMARD needs d in {64, 128};
 *              TQ_ROT_DENSE takes any multiple of 32 up to 4096.
 *   code_bits  Lloyd-Max code bits per coordinate, 1..3.
 *   kind       TQ_ROT_HADAMARD or TQ_ROT_DENSE.
 *   signs      host [d] int8 of +1/-1 (the Hadamard sign diagonal D);
 *              required for TQ_ROT_HADAMARD, ignored otherwise.
 *   gauss_pi   host [d*d] float64 row-major Gaussian draws whose QR factor
 *              (sign-fixed) is Pi; required for TQ_ROT_DENSE, else ignored.
 *   gauss_s    host [m*d] float32 row-major N(0,1) draws; each is rounded to
 *              the nearest bf16-representable value to form S.
 *   m          QJL sketch size; must equal d.
 *   rope_base  RoPE base (e.g. 10000); 0 disables RoPE for this handle.
 *   rope_max_pos  positions 0..rope_max_pos-1 are supported (ignored when
 *              rope_base is 0); at most 2^31.
 *   out        receives the handle.
 * The random draws are inputs here (tq_build_rotation_seeded draws them
 * from a seed instead).  Builds the codebook (tq_lloyd_max), Pi, S and
 * two-level RoPE tables on the host in float64 and uploads them.
 * Synchronous.
 * Returns TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_ENOMEM or TQ_ECUDA.
 */
int tq_build_rotation(int d, int code_bits, int kind, const int8_t* signs,
                      const double* gauss_pi, const float* gauss_s, int m,
                      double rope_base, int64_t rope_max_pos, tq_rotation** out);

/*
 * tq_rotation_draws - host only; the random draws a seeded handle is built
 * from.  [TurboQuant] Étape 1 and "QJL" (a random rotation, a Gaussian
 * projection S), [NSNQuant] §2 (random sign diagonal D), [TurboESM] §2.B (a
 * rotation per layer and head, reproducible from its seed).  The pages name
 * no generator; this library uses Philox4x32-10 (Salmon et al., "Parallel
 * random numbers: as easy as 1, 2, 3", SC 2011) with key = (seed mod 2^32,
 * seed >> 32) and counter = (i mod 2^32, i >> 32, stream, 0):
 *   stream 0  D_i = -1 if the top bit of word 0 of block i is set, else +1;
 *   stream 1  S, m*d Gaussians row-major; stream 2  the d*d Gaussian matrix
 *             of a dense rotation, row-major.  Gaussians come in pairs from
 *             block p: uniforms u = ((w0>>6)*2^26 + (w1>>6) + 1/2) / 2^52
 *             from words (0,1) and (2,3), then Box-Muller z_2p = r cos(2 pi
 *             u2), z_2p+1 = r sin(2 pi u2), r = sqrt(-2 ln u1), in float64.
 *   d, m        1..4096
 *   kind        TQ_ROT_HADAMARD or TQ_ROT_DENSE (gauss_pi is filled only
 *               for TQ_ROT_DENSE)
 *   signs       host out [d] int8 of +-1, or NULL
 *   gauss_pi    host out [d*d] float64, or NULL
 *   gauss_s     host out [m*d] float32 (each float64 draw rounded to the
 *               nearest float32), or NULL
 * Returns TQ_OK or TQ_EINVAL.  Pure host computation; needs no GPU.
 */
int tq_rotation_draws(int d, int kind, uint64_t seed, int m, int8_t* signs,
                      double* gauss_pi, float* gauss_s);

/*
 * tq_build_rotation_seeded - tq_build_rotation_ex from a 64-bit seed: the
 * handle built from the draws tq_rotation_draws(d, kind, seed, m, ...)
 * returns, identical to passing those draws to tq_build_rotation_ex with the
 * same residual mode.  Other arguments and statuses as tq_build_rotation.
 */
int tq_build_rotation_seeded(int d, int code_bits, int kind, int residual,
                             uint64_t seed, int m, double rope_base,
                             int64_t rope_max_pos, tq_rotation** out);

/*
 * tq_build_rotation_ex - tq_build_rotation with a choice of residual
 * correction.  residual = TQ_RES_QJL is tq_build_rotation.  residual =
 * TQ_RES_SIGN keeps one sign bit per rotated residual coordinate and the mean
 * residual magnitude e = ||r||_1 / d in place of ||r|| ([TurboESM] §2.D: the
 * residual is corrected as x~ = x^ + e sign(r); the page calibrates e, here
 * each vector's own mean magnitude is stored).  Such a handle holds S = I
 * (gauss_s is ignored and may be NULL) and the estimator constant 1, so every
 * entry point scores and accumulates sign(r) against q~ itself:
 *   score = ||x|| <q~, c[idx]> + e <q~, 2z - 1>.
 * Records keep the same layout (the signs array holds sign(r), norms[1] e).
 * Other arguments and statuses as tq_build_rotation.
 */
int tq_build_rotation_ex(int d, int code_bits, int kind, int residual,
                         const int8_t* signs, const double* gauss_pi,
                         const float* gauss_s, int m, double rope_base,
                         int64_t rope_max_pos, tq_rotation** out);

/* Release a handle and its device memory (NULL is accepted). */
int tq_free_rotation(tq_rotation* h);

/*
 * tq_rotation_export - copy the handle's tables to the host (for checks).
 *   pi          host out [d*d] float32 row-major Pi (y = Pi u), or NULL
 *   s           host out [m*d] float32 row-major S, or NULL
 *   levels      host out [2^bits] float64, or NULL
 *   thresholds  host out [2^bits - 1] float64, or NULL
 * Synchronous.  Returns TQ_OK, TQ_EINVAL or TQ_ECUDA.
 */
int tq_rotation_export(const tq_rotation* h, float* pi, float* s,
                       double* levels, double* thresholds);

/*
 * tq_tensor_core_selftest - diagnostic: runs one 128 x 128 x 128 bf16 product
 * and two 128 x 64 x 64 products (second operand K-major, and MN-major as
 * the encoder attention's value operand) through the 5th-generation
 * tensor-core path (tcgen05 with operands in swizzled shared memory and the
 * accumulator in tensor memory) on the current device, with exactly
 * representable small-integer operands, and stores in *mismatches the
 * number of result elements that differ from the exact integer products
 * (0 on a working device).  Synchronous; allocates and frees its own 64 KB
 * of device memory.  Returns TQ_OK, TQ_EINVAL, TQ_ENOMEM or TQ_ECUDA.
 */
int tq_tensor_core_selftest(int64_t* mismatches);

/*
 * tq_wait_selftest - diagnostic of the bounded waits every tensor-core and
 * TMA wait in the kernels uses: one thread initialises an mbarrier that
 * expects one arrival and waits for its first phase with a limit of 2^16
 * polls.  arrive != 0: the thread arrives first, and *completed = 1 when the
 * wait saw the phase complete.  arrive == 0: nothing completes the phase;
 * the wait gives up after its limit and *completed = 0 (the context stays
 * usable; no trap, no fault).  Synchronous; allocates and frees 4 bytes of
 * device memory.  Returns TQ_OK, TQ_EINVAL, TQ_ENOMEM or TQ_ECUDA.
 */
int tq_wait_selftest(int arrive, int* completed);

/* Record geometry of a handle: d, m, bits and bytes of codes / signs. */
int tq_rotation_dims(const tq_rotation* h, int* d, int* m, int* bits,
                     int64_t* code_bytes, int64_t* sign_bytes);

/*
 * tq_quantize_kv - encode n vectors into packed records.
 * [TurboESM] §2.A (RoPE first), [TurboQuant] Étape 1 (rotate, quantize each
 * coordinate, keep the norm) and Étape 2 + "QJL" (sign bits of S r and ||r||),
 * [TurboESM] §2.D (residual r = x - x_hat), §3 (quantize + pack at prefill).
 *   h           handle (d, bits, Pi, S, codebook, RoPE tables)
 *   x           device [n, ld] elements of `dtype` (TQ_F32 or TQ_BF16); row i
 *               is the vector; ld >= d, ld % 8 == 0 for bf16, % 4 for f32
 *   n           number of vectors (0 is a no-op)
 *   pos         device [n] int64 positions, or NULL
 *   pos_period, pos_offset   with pos == NULL, row i sits at position
 *               pos_offset + (i mod pos_period)
 *   apply_rope  nonzero: rotate by RoPE at the row's position before Pi
 *               (needs a handle built with rope_base > 0 and every position
 *               in [0, rope_max_pos))
 *   codes, signs, norms  device outputs; row i is written to record
 *               i * out_stride of each array (records of code_bytes,
 *               sign_bytes and 2 floats); codes and signs 4-byte aligned,
 *               norms 8-byte aligned
 *   out_stride  records between consecutive output rows (>= 1)
 * Positions out of range write NaN norms for that row (a host-given
 * pos_period/pos_offset out of range is rejected with TQ_EINVAL instead).
 */
int tq_quantize_kv(const tq_rotation* h, const void* x, int dtype, int64_t n,
                   int64_t ld, const int64_t* pos, int64_t pos_period,
                   int64_t pos_offset, int apply_rope, uint8_t* codes,
                   uint8_t* signs, float* norms, int64_t out_stride,
                   void* stream);

/*
 * tq_quantize_kv_pair - the keys and values one decode step appends, in one
 * call: n rows of xk with handle hk (RoPE as in tq_quantize_kv, with pos /
 * pos_period / pos_offset / apply_rope) and n rows of xv with handle hv
 * (never RoPE), both of `dtype` with row stride ld, written to record
 * i * out_stride of the K and V arrays.  Records are identical to two
 * tq_quantize_kv calls.  For n <= 256 with equal d and bits both sets are
 * encoded by one launch; otherwise the two calls run in order.
 * Returns TQ_OK, TQ_EINVAL or TQ_EUNSUPPORTED as tq_quantize_kv.
 */
int tq_quantize_kv_pair(const tq_rotation* hk, const void* xk, const tq_rotation* hv,
                        const void* xv, int dtype, int64_t n, int64_t ld,
                        const int64_t* pos, int64_t pos_period, int64_t pos_offset,
                        int apply_rope, uint8_t* k_codes, uint8_t* k_signs,
                        float* k_norms, uint8_t* v_codes, uint8_t* v_signs,
                        float* v_norms, int64_t out_stride, void* stream);

/*
 * tq_quantize_kv_scatter - tq_quantize_kv with an explicit destination record
 * per row: row i is written to record out_rows[i] of the codes, signs and
 * norms arrays.  One call writes rows bound for many sequences of a cache,
 * e.g. the flush of every sequence's full-precision window ([NSNQuant] §4,
 * "Résidus": the residual is quantized and appended when full) into records
 * T_b .. T_b + R - 1 of each sequence b, with pos giving each row's position.
 *   out_rows    device [n] int64 destination records; rows whose entry lies
 *               outside [0, n_records) are skipped (nothing written)
 *   n_records   records the codes, signs and norms arrays hold (>= 1)
 *   other arguments as in tq_quantize_kv (out_stride is not used)
 * Records are identical to tq_quantize_kv's for the same rows.  Returns the
 * statuses of tq_quantize_kv.
 */
int tq_quantize_kv_scatter(const tq_rotation* h, const void* x, int dtype,
                           int64_t n, int64_t ld, const int64_t* pos,
                           int64_t pos_period, int64_t pos_offset,
                           int apply_rope, uint8_t* codes, uint8_t* signs,
                           float* norms, const int64_t* out_rows,
                           int64_t n_records, void* stream);

/*
 * tq_quantize_kv_pair_scatter - tq_quantize_kv_pair with destination records
 * out_rows[i] for row i of both sets (keys with RoPE at pos, values without),
 * e.g. the new token of each sequence of a ragged batch appended at its own
 * length.  One launch for n <= 256 with equal d and bits, else one launch per
 * set.  Arguments as in tq_quantize_kv_pair and tq_quantize_kv_scatter.
 */
int tq_quantize_kv_pair_scatter(const tq_rotation* hk, const void* xk,
                                const tq_rotation* hv, const void* xv, int dtype,
                                int64_t n, int64_t ld, const int64_t* pos,
                                int64_t pos_period, int64_t pos_offset,
                                int apply_rope, uint8_t* k_codes,
                                uint8_t* k_signs, float* k_norms,
                                uint8_t* v_codes, uint8_t* v_signs,
                                float* v_norms, const int64_t* out_rows,
                                int64_t n_records, void* stream);

/*
 * tq_nsn_shift - the Normalize-Shift-Normalize transform of [NSNQuant] §1
 * as a shift ahead of the codec (the NSN record mode).  For each of n_blocks
 * blocks of L rows (a sequence and head), after RoPE at positions
 * pos_offset + t when apply_rope (the handle's base; [TurboESM] §2.A):
 *   s1_t = ||x~_t|| / sqrt(d),  o = mean_t x~_t / s1_t (per channel),
 *   x'_t = x~_t - s1_t o  (= s1 s2 x3 of the page: x3's direction, norm
 *          s1 s2 sqrt(d))
 * tq_quantize_kv of x' without RoPE then writes the records; s1 and o are
 * kept beside them for tq_decode_attention_nsn.
 *   h           handle (d = 64 or 128; its RoPE tables when apply_rope)
 *   x           device rows in dtype, row b*L + t at x + (b*L + t)*ld
 *   n_blocks    0 .. 65535
 *   x_shift     device [n_blocks*L, d] float32 output x' (8-byte aligned:
 *               it holds the blocks' partial sums before x')
 *   s1          device [n_blocks*L] float32 output
 *   o           device [n_blocks, d] float32 output
 * Zero rows have s1 = 0 and add nothing to o.  The block sums run in double
 * in a fixed order, so the outputs do not depend on scheduling.  Returns
 * TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED or TQ_ECUDA.
 */
int tq_nsn_shift(const tq_rotation* h, const void* x, int dtype,
                 int64_t n_blocks, int64_t L, int64_t ld, int64_t pos_offset,
                 int apply_rope, float* x_shift, float* s1, float* o,
                 void* stream);

/*
 * tq_quantize_dense - encode n vectors with a dense-rotation handle
 * (TQ_ROT_DENSE).  Same steps and record format as tq_quantize_kv, without
 * RoPE; y = Pi x and S r are dense contractions here, computed as fp32 GEMMs
 * over chunks of vectors.  [TurboQuant] "Principe", Étape 1 / Étape 2, "QJL".
 *   x           device [n, ld] float32, ld >= d, ld % 4 == 0, 16-byte aligned
 *   codes, signs, norms  device outputs, records 0..n-1 (contiguous)
 *   workspace   device scratch, 16-byte aligned; any size of at least
 *               (d + m) * 4 bytes works - vectors are processed in chunks of
 *               workspace_bytes / ((d + m) * 4); tq_quantize_dense_workspace_size
 *               gives a size that processes up to 32768 vectors per chunk
 * Returns TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED (not a dense handle),
 * TQ_EWORKSPACE or TQ_ECUDA.
 */
int tq_quantize_dense(const tq_rotation* h, const float* x, int64_t n,
                      int64_t ld, uint8_t* codes, uint8_t* signs, float* norms,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Suggested workspace bytes for tq_quantize_dense of n vectors (0 if invalid). */
size_t tq_quantize_dense_workspace_size(const tq_rotation* h, int64_t n);

/*
 * tq_search_topk - brute-force maximum-inner-product top-k from packed codes.
 * [TurboQuant] "Expériences et résultats", "Performances en recherche
 * vectorielle" (search without large codebooks) and "QJL" (the estimator):
 *   score(q, n) = ||x_n|| <Pi q, c[idx_n]> + ||r_n|| sqrt(pi/2)/m <S Pi q, sign(S r_n)>
 *   h           dense-rotation handle (d % 128 == 0)
 *   queries     device [nq, d] float32 (16-byte aligned), nq >= 1
 *   codes, signs, norms  device packed database, records 0..N-1
 *   k           1..32
 *   scores, ids device [nq, k] outputs: best first; ties go to the lower id;
 *               when N < k the tail holds -inf and id -1
 *   workspace   device scratch of tq_search_workspace_size(...) bytes,
 *               256-byte aligned
 * Returns TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EWORKSPACE or TQ_ECUDA.
 */
int tq_search_topk(const tq_rotation* h, const float* queries, int nq,
                   const uint8_t* codes, const uint8_t* signs,
                   const float* norms, int64_t N, int k, float* scores,
                   int64_t* ids, void* workspace, size_t workspace_bytes,
                   void* stream);

/* Workspace bytes tq_search_topk needs (0 if invalid). */
size_t tq_search_workspace_size(const tq_rotation* h, int nq, int64_t N, int k);

/*
 * tq_search_merge_topk - the best k of n_lists candidate lists per query,
 * e.g. the top-k lists of the database shards of a distributed search
 * ([TurboQuant] "Performances en recherche vectorielle": brute-force top-k).
 *   cand_scores, cand_ids  device [n_lists][nq][k] (float32, int64), each
 *               list best first as tq_search_topk writes them (entries with
 *               id -1 or score -inf are ignored)
 *   id_offsets  device [n_lists] int64 added to the ids of each list (the
 *               shard's first global row), or NULL
 *   scores, ids device [nq][k] outputs: best first, ties to the lower id,
 *               -inf / -1 when fewer than k candidates exist
 * Returns TQ_OK, TQ_EINVAL or TQ_ECUDA.
 */
int tq_search_merge_topk(const float* cand_scores, const int64_t* cand_ids,
                         int n_lists, int nq, int k, const int64_t* id_offsets,
                         float* scores, int64_t* ids, void* stream);

/*
 * tq_decode_attention - one decode step of attention over packed K/V caches.
 * [TurboESM] §2.E: dequantization, residual correction, inverse rotation
 * Pi^T and an online softmax fused in one pass over the cache;
 * [TurboQuant] "QJL": score <q, x_hat> + ||r|| sqrt(pi/2)/m <S q, sign(S r)>.
 *   hk, hv      handles of the K and V caches (d = 128 for both; hk carries
 *               RoPE, hv must not apply RoPE to V - its rope base is unused)
 *   q           device [B, Hq, d] elements of q_dtype
 *   q_pos       device [B] int64 query positions (used when hk has RoPE)
 *   k_codes, k_signs, k_norms, v_codes, v_signs, v_norms
 *               device caches; sequence (b, kv-head j) occupies records
 *               (b*Hkv + j)*cache_stride .. + T-1; all 16-byte aligned
 *   cache_stride  records between consecutive sequences (>= T, even)
 *   B, Hq, Hkv  batch, query heads, KV heads; Hq % Hkv == 0,
 *               Hq/Hkv in {1, 2, 4, 8} and B*Hkv <= 65535
 *   T           cached tokens per sequence, or with seq_lens the largest
 *               length (0 gives an all-zero output)
 *   seq_lens    device [B] int32 tokens of each sequence b (records 0 ..
 *               seq_lens[b]-1 of its KV heads), each in 0..T; NULL: all T.
 *               A length outside 0..T makes that sequence's outputs NaN
 *               (device memory is not read on the host)
 *   scale       softmax scale (typically 1/sqrt(d))
 *   out         device [B, Hq, d] float32
 *   workspace   device scratch of at least tq_decode_workspace_size(...)
 *               bytes, 256-byte aligned; contents need no initialisation
 * Query head h reads KV head h / (Hq/Hkv).  Returns TQ_OK, TQ_EINVAL,
 * TQ_EUNSUPPORTED, TQ_EWORKSPACE or TQ_ECUDA.
 */
int tq_decode_attention(const tq_rotation* hk, const tq_rotation* hv,
                        const void* q, int q_dtype, const int64_t* q_pos,
                        const uint8_t* k_codes, const uint8_t* k_signs,
                        const float* k_norms, const uint8_t* v_codes,
                        const uint8_t* v_signs, const float* v_norms,
                        int64_t cache_stride, int B, int Hq, int Hkv, int64_t T,
                        const int32_t* seq_lens, float scale, float* out,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * tq_decode_attention_nsn - tq_decode_attention over records written in the
 * NSN mode (tq_nsn_shift, then tq_quantize_kv of the shifted rows):
 * [NSNQuant] §1 and §4, "the attention score uses s1, s2, o directly".  Key t
 * of a sequence stands for k'_t + s1k_t o_k and value t for v'_t + s1v_t o_v
 * (k', v' the records' vectors), so
 *   score_t = scale (<q', k'^_t> + s1k_t <q', o_k>),
 *   out     = sum_t p_t v'^_t + o_v sum_t p_t s1v_t.
 *   k_s1, v_s1  device float32 s1 of every record, indexed as the norms
 *               ((b*Hkv + j)*cache_stride + t); 16-byte aligned
 *   k_o, v_o    device [B*Hkv, d] float32 shifts (keys: after RoPE)
 *   cache_stride  as tq_decode_attention, and a multiple of 4
 *   other arguments and the workspace as tq_decode_attention
 * Returns TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EWORKSPACE or TQ_ECUDA.
 */
int tq_decode_attention_nsn(const tq_rotation* hk, const tq_rotation* hv,
                            const void* q, int q_dtype, const int64_t* q_pos,
                            const uint8_t* k_codes, const uint8_t* k_signs,
                            const float* k_norms, const uint8_t* v_codes,
                            const uint8_t* v_signs, const float* v_norms,
                            const float* k_s1, const float* k_o,
                            const float* v_s1, const float* v_o,
                            int64_t cache_stride, int B, int Hq, int Hkv,
                            int64_t T, const int32_t* seq_lens, float scale,
                            float* out, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * tq_decode_attention_append - one decode step with the new token's key and
 * value appended to the caches first, in the same launch as the query
 * preparation: [NSNQuant] §4 ("Résidus": quantize the new token and append
 * it), then tq_decode_attention over caches that now hold it.
 *   k_new, v_new  device [B*Hkv, d] rows in q_dtype, row b*Hkv + j the new
 *               key / value of sequence b, KV head j; the key takes RoPE at
 *               position q_pos[b] (when hk has RoPE)
 *   k_codes .. v_norms  the caches (written: record len_b - 1 of each
 *               sequence, len_b = seq_lens[b] or T, which counts the new
 *               token; nothing is written where len_b is 0 or outside 0..T)
 *   other arguments and the workspace as tq_decode_attention
 * Same result as tq_quantize_kv_pair of the new rows into those records
 * followed by tq_decode_attention.  Returns TQ_OK, TQ_EINVAL,
 * TQ_EUNSUPPORTED, TQ_EWORKSPACE or TQ_ECUDA.
 */
int tq_decode_attention_append(const tq_rotation* hk, const tq_rotation* hv,
                               const void* q, int q_dtype,
                               const int64_t* q_pos, const void* k_new,
                               const void* v_new, uint8_t* k_codes,
                               uint8_t* k_signs, float* k_norms,
                               uint8_t* v_codes, uint8_t* v_signs,
                               float* v_norms, int64_t cache_stride, int B,
                               int Hq, int Hkv, int64_t T,
                               const int32_t* seq_lens, float scale,
                               float* out, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * tq_decode_attention_nsn_append - tq_decode_attention_append over NSN
 * records: [NSNQuant] §1 and §4 (a token after the block keeps the block's
 * statistics).  The new key takes RoPE at q_pos[b]; each new row x~ then
 * gets s1 = ||x~|| / sqrt(d), written to k_s1 / v_s1 at record len_b - 1,
 * and its record is that of x' = x~ - s1 o with its sequence's o (k_o / v_o,
 * not changed).  Then tq_decode_attention_nsn over the caches that now hold
 * the token.
 *   k_s1, v_s1  device float32 s1 arrays as tq_decode_attention_nsn (written
 *               at the new records); 16-byte aligned
 *   k_o, v_o    device [B*Hkv, d] float32 shifts (keys: after RoPE)
 *   cache_stride  a multiple of 4 (and even)
 *   other arguments as tq_decode_attention_append
 * Returns TQ_OK, TQ_EINVAL (also for any of the four side arrays missing),
 * TQ_EUNSUPPORTED, TQ_EWORKSPACE or TQ_ECUDA.
 */
int tq_decode_attention_nsn_append(const tq_rotation* hk, const tq_rotation* hv,
                                   const void* q, int q_dtype,
                                   const int64_t* q_pos, const void* k_new,
                                   const void* v_new, uint8_t* k_codes,
                                   uint8_t* k_signs, float* k_norms,
                                   uint8_t* v_codes, uint8_t* v_signs,
                                   float* v_norms, float* k_s1,
                                   const float* k_o, float* v_s1,
                                   const float* v_o, int64_t cache_stride,
                                   int B, int Hq, int Hkv, int64_t T,
                                   const int32_t* seq_lens, float scale,
                                   float* out, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Workspace bytes tq_decode_attention needs for these sizes (0 if invalid). */
size_t tq_decode_workspace_size(const tq_rotation* hk, const tq_rotation* hv,
                                int B, int Hq, int Hkv, int64_t T);

/*
 * tq_decode_attention_window - tq_decode_attention over a packed cache plus
 * a full-precision window of the most recent tokens.
 * [NSNQuant] §4, "Résidus" (after KIVI): the cache is a quantized part and a
 * residual kept in full precision; when the residual is full the caller
 * flushes it (tq_quantize_kv / tq_quantize_kv_pair with positions T .. T+R-1
 * into records T .. T+R-1) and empties the window.
 *   hk ... cache_stride, B, Hq, Hkv, T, seq_lens, scale, out
 *               as in tq_decode_attention (T packed tokens, possibly 0; with
 *               seq_lens, sequence b has seq_lens[b] packed tokens and its
 *               window tokens sit at positions seq_lens[b] + i)
 *   k_window, v_window
 *               device [B*Hkv, window_stride, d] elements of window_dtype:
 *               row (b*Hkv + j)*window_stride + i is token i of the window
 *               of sequence b, KV head j - the key as the model produced it
 *               (before RoPE) and its value; token i sits at position T + i,
 *               where its key gets RoPE when hk has a RoPE base (T + R must
 *               not exceed the handle's rope_max_pos)
 *   window_dtype  TQ_F32 or TQ_BF16 (both pointers 16-byte aligned)
 *   window_stride rows between consecutive sequences' windows (>= R)
 *   R           window tokens, 0 .. 1024 (0 gives tq_decode_attention's
 *               result exactly)
 *   workspace   at least tq_decode_window_workspace_size(...) bytes
 * The softmax runs over all T + R tokens: scores of window tokens are
 * <RoPE(q, q_pos), RoPE(k_i, T + i)> * scale in fp32, their values enter
 * unquantized.  Returns TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED (R > 1024 or as
 * tq_decode_attention), TQ_EWORKSPACE or TQ_ECUDA.
 */
int tq_decode_attention_window(const tq_rotation* hk, const tq_rotation* hv,
                               const void* q, int q_dtype, const int64_t* q_pos,
                               const uint8_t* k_codes, const uint8_t* k_signs,
                               const float* k_norms, const uint8_t* v_codes,
                               const uint8_t* v_signs, const float* v_norms,
                               int64_t cache_stride, const void* k_window,
                               const void* v_window, int window_dtype,
                               int64_t window_stride, int R, int B, int Hq,
                               int Hkv, int64_t T, const int32_t* seq_lens,
                               float scale, float* out, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Workspace bytes tq_decode_attention_window needs (0 if invalid). */
size_t tq_decode_window_workspace_size(const tq_rotation* hk,
                                       const tq_rotation* hv, int B, int Hq,
                                       int Hkv, int64_t T, int R);

/*
 * tq_decode_partials - tq_decode_attention up to, but not including, the
 * final normalisation: for every query head, the partial record of the
 * softmax over this call's tokens, so that calls over disjoint token ranges
 * of the same sequences (e.g. the shards of a long context on several GPUs)
 * can be combined later by tq_decode_merge_partials.  [TurboESM] §2.E (the
 * fused pass: online softmax, value accumulation in the rotated space,
 * Pi^T at the end); the split into partials is the log-sum-exp rule of an
 * online softmax, which the merge applies exactly.
 *   hk ... seq_lens, scale  as in tq_decode_attention (the records are the
 *               caller's shard; positions are those the keys were encoded
 *               with, and q_pos is the query's own position)
 *   partials    device out [B*Hq][2 + 2*d] float32: per query head (row
 *               b*Hq + h) the log2-domain max m of its logits * scale *
 *               log2(e), the sum l of 2^(logit - m), and the rotated-space
 *               sums O_code[d] and O_z[d] (value codes and QJL signs, each
 *               weighted by 2^(logit - m) and the record's norm).  A shard
 *               without tokens gives m = -inf, l = 0, zeros.
 *   workspace   as for tq_decode_attention with the same sizes
 * Returns the statuses of tq_decode_attention.
 */
int tq_decode_partials(const tq_rotation* hk, const tq_rotation* hv,
                       const void* q, int q_dtype, const int64_t* q_pos,
                       const uint8_t* k_codes, const uint8_t* k_signs,
                       const float* k_norms, const uint8_t* v_codes,
                       const uint8_t* v_signs, const float* v_norms,
                       int64_t cache_stride, int B, int Hq, int Hkv, int64_t T,
                       const int32_t* seq_lens, float scale, float* partials,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * tq_decode_merge_partials - the attention output from n_parts partial
 * records per query head (tq_decode_partials over disjoint token ranges):
 * log-sum-exp combination, the QJL value correction sqrt(pi/2)/m S^T O_z and
 * Pi^T of the value handle, divided by the combined sum.  [TurboESM] §2.E;
 * [TurboQuant] "QJL".
 *   hv          value handle (d = 128, Hadamard)
 *   partials    device [n_parts][B*Hq][2 + 2*d] float32 (part-major, e.g.
 *               the all-gather of every rank's tq_decode_partials output)
 *   n_parts     1 .. 65536; the merge keeps n_parts * G floats of weights
 *               in shared memory, so TQ_EUNSUPPORTED past the device's
 *               per-block limit (about 5,900 parts at G = 8 on B200)
 *   B, Hq, Hkv  as in tq_decode_attention
 *   out         device [B, Hq, d] float32
 * Returns TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED or TQ_ECUDA.
 */
int tq_decode_merge_partials(const tq_rotation* hv, const float* partials,
                             int n_parts, int B, int Hq, int Hkv, float* out,
                             void* stream);

/*
 * tq_encoder_attention - bidirectional attention of S queries per head over
 * a packed K/V cache (prefill / encoder use).
 * [TurboESM] §2.A (RoPE before the rotation, so (Pi R_i q)^T (Pi R_j k) keeps
 * the attention score), §2.E (dequantization, residual correction, Pi^T and
 * the softmax fused); [TurboQuant] "QJL" (the score estimator).
 *   hk, hv      handles of K and V (same d in {64, 128}, same bits, Hadamard)
 *   q           device [B, Hq, S, d] of q_dtype; query s sits at position
 *               q_pos_offset + s (RoPE when hk has a RoPE base; every such
 *               position must be below rope_max_pos)
 *   caches      as in tq_decode_attention: sequence (b, j) at records
 *               (b*Hkv + j)*cache_stride .. + T-1, 16-byte aligned arrays
 *   B, Hq, Hkv  Hq % Hkv == 0 (query head h reads KV head h / (Hq/Hkv))
 *   S, T        queries per head (>= 1) and cached keys per sequence (>= 0)
 *   scale       softmax scale
 *   out         device [B, Hq, S, d] float32
 *   workspace   device scratch of tq_encoder_workspace_size(...) bytes,
 *               256-byte aligned
 * No mask: every query sees all T keys.  Returns TQ_OK, TQ_EINVAL,
 * TQ_EUNSUPPORTED, TQ_EWORKSPACE or TQ_ECUDA.
 */
int tq_encoder_attention(const tq_rotation* hk, const tq_rotation* hv,
                         const void* q, int q_dtype, int64_t q_pos_offset,
                         const uint8_t* k_codes, const uint8_t* k_signs,
                         const float* k_norms, const uint8_t* v_codes,
                         const uint8_t* v_signs, const float* v_norms,
                         int64_t cache_stride, int B, int Hq, int Hkv, int S,
                         int64_t T, float scale, float* out, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Workspace bytes tq_encoder_attention needs (0 if invalid). */
size_t tq_encoder_workspace_size(const tq_rotation* hk, int B, int Hq, int S);

/*
 * tq_decode_attention_noalloc - tq_decode_attention for callers that cannot
 * allocate device memory.  The pages have no counterpart; this entry point
 * is a deployment convenience.
 * Callers such as serving runtimes that fix their device memory budget up
 * front and forbid cudaMalloc afterwards, or plugin hosts that give the
 * library no allocator, cannot supply the `workspace` of
 * tq_decode_attention.  This variant takes the same arguments minus the
 * workspace and uses instead a fixed 16 MiB scratch array compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.  It calls no allocating routine.
 *   - Sizes whose tq_decode_workspace_size(...) exceeds 16 MiB are rejected
 *     with TQ_EWORKSPACE before anything is launched (e.g. batch 16 x 8 KV
 *     heads x 32768 tokens with 4 query heads per KV head needs ~6 MB).
 *   - The first call on each device looks up that device's copy of the
 *     scratch array (cudaGetSymbolAddress) with that device current; make
 *     that first call before any stream capture on the device.
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents (every call rewrites what it reads, and clears what
 *     must start at zero).  Calls whose kernels may overlap on the GPU -
 *     concurrent streams, or host threads racing on one device - race on
 *     the scratch: serialise them.
 * Returns the statuses of tq_decode_attention, in this order: the handle and
 * size checks (TQ_EINVAL, TQ_EUNSUPPORTED), then TQ_EWORKSPACE for sizes
 * beyond the scratch, then the pointer checks and launches.
 */
int tq_decode_attention_noalloc(const tq_rotation* hk, const tq_rotation* hv,
                                const void* q, int q_dtype, const int64_t* q_pos,
                                const uint8_t* k_codes, const uint8_t* k_signs,
                                const float* k_norms, const uint8_t* v_codes,
                                const uint8_t* v_signs, const float* v_norms,
                                int64_t cache_stride, int B, int Hq, int Hkv,
                                int64_t T, const int32_t* seq_lens, float scale,
                                float* out, void* stream);

/*
 * tq_profile_next_decode - instrumentation for benchmarks.  The next
 * tq_decode_attention call made by this host thread records `ev_begin`
 * immediately before and `ev_end` immediately after its split-KV kernel, on
 * that call's stream, so the caller can time the dominant kernel alone with
 * cudaEventElapsedTime.  Both are cudaEvent_t passed as void* (created by the
 * caller, on the handle's device); NULL, NULL cancels.  One-shot: consumed by
 * the next call (also when that call fails).  Returns TQ_OK or TQ_EINVAL.
 */
int tq_profile_next_decode(void* ev_begin, void* ev_end);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
