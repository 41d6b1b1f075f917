/*
 * tq.h — C ABI of the B200 compressed-KV library (libtq.so).
 *
 * The library computes the TurboQuant / TurboESM key-value cache path:
 *   RoPE -> orthogonal rotation Pi -> per-vector fp32 norm + b-bit Lloyd-Max
 *   index per coordinate -> (keys) 1-bit QJL sign sketch of the residual plus
 *   the residual norm -> attention computed directly over the packed cache.
 * Sources: gist.science "TurboESM: Ultra-Efficient 3-Bit KV Cache Quantization
 * for Protein Language Models with Orthogonal Rotation and QJL Correction"
 * (technical summary, sections 2A-2E) and 7minutos.es "KV cache está
 * consumiendo tu VRAM ... TurboQuant" (Etapa 1 and Etapa 2).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers documented "device" must point to memory of the current CUDA
 *    device; "host" pointers to ordinary host memory. The caller owns every
 *    buffer; the library allocates nothing.
 *  - Every GPU call is asynchronous on the given stream (`stream` is a
 *    cudaStream_t passed as void*; NULL = legacy default stream).
 *  - Arguments are validated on the host; on any violation the call returns
 *    TQ_ERR_INVALID_ARG (or TQ_ERR_UNSUPPORTED) without launching anything.
 *    tq_last_error_string() then describes the problem (per host thread).
 *  - Kernels never trap. Conditions only the device can see are OR-ed into
 *    the optional device word *d_status (TQ_DEV_* bits); read it after the
 *    stream has synchronised. A NULL d_status disables that reporting.
 *  - Pi and S are data (seeded by the caller); the library draws no random
 *    numbers.
 *
 * Packed-cache layout (one "row" per vector, rows of a plane are contiguous)
 * -------------------------------------------------------------------------
 *  index plane  uint8  [n][d*bits/8]   8 coordinates per `bits` bytes; the
 *               group of coordinates 8g..8g+7, read as a little-endian integer,
 *               holds code[8g+j] at bits [bits*j, bits*j+bits).
 *  sign plane   uint32 [n][ceil(d/32)] (keys) bit i of the sketch at bit
 *               (i mod 32) of word i/32; pad bits are 0.
 *  norm plane   float  [n]             ||x|| of the (RoPE'd) input vector.
 *  rnorm plane  float  [n]             (keys) ||r||, r = Pi x - ||x|| c[code].
 * A cache for [B][H][N] vectors stores row (b*H + h)*ctx_stride + t.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or combination   */
  TQ_ERR_UNSUPPORTED = 2,   /* valid request the library does not implement  */
  TQ_ERR_CUDA = 3,          /* a CUDA runtime call failed (see error string)  */
  TQ_ERR_WORKSPACE = 4      /* workspace missing or smaller than required    */
} tq_status;

/* Device-side status bits OR-ed into *d_status. */
#define TQ_DEV_BAD_CODEBOOK   0x1  /* boundaries not strictly increasing       */
#define TQ_DEV_BAD_POSITION   0x2  /* a RoPE position was negative            */
#define TQ_DEV_TIMEOUT        0x4  /* a kernel gave up waiting on its own pipeline
                                      (bounded wait); outputs of that call are invalid.
                                      The pipeline waits of the tensor-core kernels
                                      give up after 2 s, or after the number of ns in
                                      the environment variable TQ_TEST_WAIT_NS (read
                                      at each call; for tests of this path). */

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

/* Shape of one head's packed vectors. d: head dim, a multiple of 8 in
 * [8, 256]; key_bits / value_bits: index bits per coordinate, 2..4. */
typedef struct {
  int32_t d;
  int32_t key_bits;
  int32_t value_bits;
} tq_layout;

/* The planes of one packed tensor (all device pointers; 16-byte aligned).
 * sign and rnorm are used for keys only and may be NULL for values. */
typedef struct {
  uint8_t*  idx;
  uint32_t* sign;
  float*    norm;
  float*    rnorm;
} tq_planes;

/* ------------------------------------------------------------------------
 * Sizes of the packed layout.
 * ---------------------------------------------------------------------- */
/* Bytes of one index row: d*bits/8. */
int64_t tq_idx_row_bytes(int32_t d, int32_t bits);
/* 32-bit words of one sign row: ceil(d/32). */
int64_t tq_sign_words(int32_t d);
/* Total packed bytes of n vectors (index + sign + norm + rnorm planes for a
 * key, index + norm planes for a value). -1 on invalid arguments. */
int64_t tq_packed_bytes(const tq_layout* layout, int64_t n_vectors, int32_t is_key);

/* ------------------------------------------------------------------------
 * tq_make_codebook — Lloyd-Max levels for one coordinate (host only).
 *
 * 7minutos.es "KV cache ... TurboQuant", Etapa 1: after a random rotation a
 * coordinate x of a unit vector follows x^2 ~ Beta(1/2, (d-1)/2), density
 * proportional to (1-x^2)^((d-3)/2) on [-1,1]; Lloyd-Max alternates
 * "boundary = midpoint of adjacent levels" and "level = mean of its cell"
 * until the error stops improving; the codebook depends only on (d, bits).
 * gist.science TurboESM section 2C: K and V get separate tables fitted to
 * their own post-rotation coordinates ("dual LUT") — mode 1.
 *
 *  d            >= 3 (mode 0); ignored for mode 1
 *  bits         1..4 (2^bits levels)
 *  mode         0 = analytic law above; 1 = empirical Lloyd on `samples`
 *  samples      host, n_samples floats (mode 1 only; coordinates of rotated
 *               unit vectors); NULL for mode 0
 *  centroids    host out, 2^bits floats, strictly increasing
 *  boundaries   host out, 2^bits - 1 floats, midpoints of adjacent centroids
 *               (computed in double, then rounded)
 *  mse_out      host out (nullable): per-coordinate distortion (mode 0: under
 *               the law; mode 1: over the samples)
 * Start: the 2^bits equiprobable quantiles. Stop: no level moves by 1e-13
 * (mode 0; the result is then made exactly symmetric) or no sample changes
 * cell (mode 1). Errors: TQ_ERR_INVALID_ARG.
 * ---------------------------------------------------------------------- */
tq_status tq_make_codebook(int32_t d, int32_t bits, int32_t mode,
                           const float* samples, int64_t n_samples,
                           float* centroids, float* boundaries, double* mse_out);

/* ------------------------------------------------------------------------
 * tq_quantize_kv — quantise and pack n vectors (one launch; device).
 *
 * gist.science TurboESM section 2A: RoPE first, then the orthogonal Pi.
 * 7minutos.es Etapa 1: y = Pi x, each coordinate of y/||x|| replaced by the
 * index of its Lloyd-Max level. Etapa 2 (keys): the residual of stage 1 is
 * multiplied by the Gaussian S; the signs of the result (1 bit each) and the
 * residual's L2 norm are stored.
 *
 * Per vector v (row v of x):
 *   x'   = RoPE(x_v, positions[v])   rotate-half pairs (i, i+d/2) turned by
 *                                    positions[v] * rope_base^(-2i/d);
 *                                    skipped when positions==NULL or
 *                                    rope_base <= 0
 *   y    = Pi_g x'                   g = v / vectors_per_pi
 *   code_i = #{ j : y_i > ||x'|| * boundaries[j] }   (ties go to the lower code)
 *   keys: r = y - ||x'|| centroids[code];  sign_i = ((S r)_i >= 0)
 * Codes and signs equal those of exact arithmetic: any coordinate (or sign)
 * whose fp32 margin is within a guard band of its decision is recomputed in
 * fp64 before it is stored. Calls of at most 1024 vectors with one shared Pi
 * run entirely in fp64, one CTA per vector (the kernel of tq_append_kv).
 *
 *  layout          d and the bits of this tensor (key_bits if is_key, else
 *                  value_bits)
 *  is_key          1: keys (signs + rnorm written, S required); 0: values
 *  x               device, n_vectors rows of d elements of x_dtype
 *                  (TQ_F32 or TQ_BF16), row v at x + v*row_stride elements
 *  positions       device int32 [n_vectors] or NULL
 *  Pi              device float, row-major d x d matrices; matrix g at
 *                  Pi + g*pi_stride (pi_stride 0 = one shared matrix)
 *  vectors_per_pi  rows sharing one Pi (>= 1; ignored when pi_stride == 0)
 *  S               device float d x d, row-major (keys; NULL for values)
 *  centroids, boundaries   device float, 2^bits and 2^bits-1 entries
 *  out             planes to write, n_vectors rows each (pointers device)
 *  d_status        device int32 (nullable), see TQ_DEV_*
 * Supported d: 64, 128, 200 (others: TQ_ERR_UNSUPPORTED).
 * ---------------------------------------------------------------------- */
tq_status tq_quantize_kv(const tq_layout* layout, int32_t is_key,
                         const void* x, tq_dtype x_dtype, int64_t n_vectors, int64_t row_stride,
                         const int32_t* positions, float rope_base,
                         const float* Pi, int64_t vectors_per_pi, int64_t pi_stride,
                         const float* S,
                         const float* centroids, const float* boundaries,
                         const tq_planes* out,
                         int32_t* d_status, void* stream);

/* ------------------------------------------------------------------------
 * tq_append_kv — quantise one new vector per stream into its cache slot
 * (one launch; device).
 *
 * 7minutos.es "KV cache ... TurboQuant" Etapa 1: a token's indices are
 * computed once, when it enters the cache, and stay there until it is
 * evicted; gist.science TurboESM section 2A: RoPE at the token's position
 * before the rotation. The arithmetic is that of tq_quantize_kv with one
 * shared Pi; only the destination differs: row s of x (stream s = b * hkv +
 * kv) is written to cache row s * ctx_stride + slot, the layout that
 * tq_decode_attention reads with the same ctx_stride.
 *
 *  x            device, n_streams rows of d elements (TQ_F32 or TQ_BF16),
 *               row s at x + s*row_stride elements
 *  positions    device int32 [n_streams] RoPE positions, or NULL (no RoPE)
 *  Pi, S        device float d x d (S: keys only)
 *  cache        planes of n_streams * ctx_stride rows (device pointers)
 *  slot         0 <= slot < ctx_stride; rows at other slots are not touched
 * Errors: TQ_ERR_INVALID_ARG (NULL pointers, slot out of range, strides),
 * TQ_ERR_UNSUPPORTED (d not 64, 128 or 200), TQ_ERR_CUDA.
 * ---------------------------------------------------------------------- */
tq_status tq_append_kv(const tq_layout* layout, int32_t is_key,
                       const void* x, tq_dtype x_dtype, int64_t n_streams, int64_t row_stride,
                       const int32_t* positions, float rope_base,
                       const float* Pi, const float* S,
                       const float* centroids, const float* boundaries,
                       const tq_planes* cache, int64_t ctx_stride, int64_t slot,
                       int32_t* d_status, void* stream);

/* ------------------------------------------------------------------------
 * tq_decode_attention — attention of queries over a packed K/V cache.
 *
 * gist.science TurboESM section 2E: one fused kernel unpacks the 3-bit
 * codes, applies the QJL correction, the inverse rotation Pi^T and an
 * online-softmax attention, with no dequantised intermediate in memory.
 * 7minutos.es Etapa 2: the sign bits enter through S^T scaled by
 * sqrt(pi/2)/d and the residual norm.
 *
 * For query row (b, h, n) and its KV head kv = h / (hq/hkv):
 *   q'    = RoPE(q[b,h,n], q_positions[b*nq + n])   (if enabled)
 *   q_rot = Pi_K[kv] q',   s = S q_rot
 *   score_t = scale * ( knorm_t <q_rot, cK[code_t]>
 *                       + sqrt(pi/2)/d * rnorm_t <s, 2*sign_t - 1> )
 *   out[b,h,n] = Pi_V[kv]^T sum_t softmax(score)_t vnorm_t cV[vcode_t]
 * No mask: every query attends all n_ctx tokens.
 *
 *  q          device [batch][hq][nq][d] of q_dtype (TQ_F32/TQ_BF16)
 *  nq         queries per head (1 for decode; up to n_ctx for a full
 *             bidirectional pass)
 *  q_positions device int32 [batch][nq] or NULL; rope_base <= 0 disables RoPE
 *  k, v       planes of [batch][hkv] streams; stream (b, kv) starts at row
 *             (b*hkv + kv)*ctx_stride; ctx_stride >= n_ctx (0 means n_ctx)
 *  PiK, PiV   device float d x d; matrix of KV head kv at Pi + kv*pi_stride
 *             (pi_stride 0 = shared)
 *  S          device float d x d; cK, cV device centroid tables
 *  scale      softmax scale (1/sqrt(d) in the method)
 *  out        device [batch][hq][nq][d] of out_dtype
 *  scores_out device float [batch][hq][nq][n_ctx] or NULL (raw scores, for
 *             testing; slows the call)
 *  workspace  device scratch of tq_decode_workspace_bytes() bytes
 *             (256-byte aligned); contents need no initialisation
 * ---------------------------------------------------------------------- */
tq_status tq_decode_attention(const tq_layout* layout,
                              const void* q, tq_dtype q_dtype,
                              int32_t batch, int32_t hq, int32_t hkv, int32_t nq, int64_t n_ctx,
                              int64_t ctx_stride,
                              const int32_t* q_positions, float rope_base,
                              const tq_planes* k, const tq_planes* v,
                              const float* PiK, const float* PiV, int64_t pi_stride,
                              const float* S, const float* cK, const float* cV, float scale,
                              void* out, tq_dtype out_dtype, float* scores_out,
                              void* workspace, size_t workspace_bytes,
                              int32_t* d_status, void* stream);

/* Scratch bytes tq_decode_attention needs for this shape (0 on bad args). */
size_t tq_decode_workspace_bytes(const tq_layout* layout, int32_t batch, int32_t hq, int32_t hkv,
                                 int32_t nq, int64_t n_ctx);

/* ------------------------------------------------------------------------
 * tq_decode_attention_noalloc — tq_decode_attention without a caller
 * workspace. (No counterpart in the method's description; it exists for
 * callers that cannot allocate device memory at call time — a serving loop
 * that must not stall on cudaMalloc's implicit device synchronisation, or a
 * plugin inside a host framework that owns every device allocation.)
 *
 * Arguments and results are those of tq_decode_attention minus
 * workspace/workspace_bytes. The split-KV scratch is a fixed 64 MiB device
 * array inside libtq.so (every GPU that loads the library holds it until the
 * process exits); shapes whose tq_decode_workspace_bytes() exceeds 64 MiB are
 * rejected with TQ_ERR_UNSUPPORTED and a message. The function itself calls
 * no cudaMalloc/cudaFree and no allocating routine.
 *  - The first call on each device looks the array's device address up
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture. The address is cached per device ordinal and
 *    belongs to the device's primary context (the runtime API's): callers
 *    that drive the device through their own driver-API contexts must make
 *    the primary context current for these calls.
 *  - All calls share the one array and leave their data in it. Nothing needs
 *    clearing between calls, but calls that overlap on the GPU (other streams
 *    or host threads) race on it: serialise them.
 * ---------------------------------------------------------------------- */
tq_status tq_decode_attention_noalloc(const tq_layout* layout,
                                      const void* q, tq_dtype q_dtype,
                                      int32_t batch, int32_t hq, int32_t hkv, int32_t nq, int64_t n_ctx,
                                      int64_t ctx_stride,
                                      const int32_t* q_positions, float rope_base,
                                      const tq_planes* k, const tq_planes* v,
                                      const float* PiK, const float* PiV, int64_t pi_stride,
                                      const float* S, const float* cK, const float* cV, float scale,
                                      void* out, tq_dtype out_dtype, float* scores_out,
                                      int32_t* d_status, void* stream);

/* ------------------------------------------------------------------------
 * tq_dequantize — reconstruct vectors from their planes (device).
 *
 * 7minutos.es Etapa 1: look each index up in the codebook and multiply by
 * the transpose of the rotation, K_hat = Pi^T ||x|| c[code]. Etapa 2:
 * K_tilde = K_hat + sqrt(pi/2)/d * ||r|| * Pi^T S^T (2*sign - 1)  (keys; S acts
 * in rotated coordinates, so the correction is turned back by Pi^T too).
 *
 *  planes     rows 0..n_vectors-1 (sign/rnorm read only if is_key)
 *  Pi, vectors_per_pi, pi_stride   as in tq_quantize_kv
 *  out        device, n_vectors rows of d elements of out_dtype, row v at
 *             out + v*out_stride elements
 * ---------------------------------------------------------------------- */
tq_status tq_dequantize(const tq_layout* layout, int32_t is_key, int64_t n_vectors,
                        const tq_planes* planes,
                        const float* Pi, int64_t vectors_per_pi, int64_t pi_stride,
                        const float* S, const float* centroids,
                        void* out, tq_dtype out_dtype, int64_t out_stride, void* stream);

/* ------------------------------------------------------------------------
 * tq_dequantize_sign_mean — reconstruct with TurboESM's one-bit residual
 * correction (device).
 *
 * gist.science TurboESM section 2D: only the sign of each residual
 * coordinate is stored beside the 3-bit index, and decoding adds a first-order
 * correction with the pre-calibrated mean residual magnitude e_bar:
 *   x_tilde = Pi^T ||x|| ( c[code] + e_bar (2*sign - 1) ).
 * The signs are those tq_quantize_kv writes with is_key = 1 and S = the d x d
 * identity (sign_i = (r_i >= 0), r the rotated residual); e_bar comes from
 * tq_residual_mean. A vector then needs its codes, d sign bits and ||x||
 * (36 bytes at d = 64, 3 bits; the rnorm plane is not read).
 *
 *  is_key     selects the layout's bits (key_bits or value_bits)
 *  planes     idx, sign and norm of rows 0..n_vectors-1
 *  e_bar      >= 0, in unit-vector coordinates
 *  Pi, vectors_per_pi, pi_stride, out, out_dtype, out_stride as tq_dequantize
 * Errors: TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED (n_vectors >= 2^31), TQ_ERR_CUDA.
 * ---------------------------------------------------------------------- */
tq_status tq_dequantize_sign_mean(const tq_layout* layout, int32_t is_key, int64_t n_vectors,
                                  const tq_planes* planes, const float* Pi, int64_t vectors_per_pi,
                                  int64_t pi_stride, const float* centroids, float e_bar,
                                  void* out, tq_dtype out_dtype, int64_t out_stride, void* stream);

/* ------------------------------------------------------------------------
 * tq_residual_mean — calibrate e_bar for tq_dequantize_sign_mean (host).
 *
 * gist.science TurboESM section 2D ("mean residual magnitude, calibrated
 * beforehand"): e_bar = mean over the samples u of |u - c[code(u)]|, with
 * code(u) = #{j : u > boundaries[j]}. The samples are coordinates of rotated
 * unit vectors, e.g. from tq_rotate_normalize on calibration data.
 *
 *  samples   host float [n_samples]
 *  centroids, boundaries   host float, 2^bits and 2^bits - 1 entries
 *  e_bar     host out
 * Errors: TQ_ERR_INVALID_ARG.
 * ---------------------------------------------------------------------- */
tq_status tq_residual_mean(const float* samples, int64_t n_samples, const float* centroids,
                           const float* boundaries, int32_t bits, double* e_bar);

/* ------------------------------------------------------------------------
 * tq_search_topk — k best corpus vectors per query by estimated inner product.
 *
 * sudonull.com "TurboQuant: compresión 6x de LLM KV-cache" and news.hada.io's
 * TurboQuant summary: the same codes serve vector search (recall of the true
 * top inner products among the approximate top-k). Score of corpus vector x
 * (quantised as a key: codes, signs, ||x||, ||r||) for query q:
 *   est = ||x|| <Pi q, c[code_x]> + sqrt(pi/2)/d ||r_x|| <S Pi q, 2 sign_x - 1>
 * Ranking: decreasing est; equal scores by increasing corpus index.
 *
 *  q           device [n_queries][d] of q_dtype
 *  db          key planes of n_db corpus vectors (layout.key_bits bits)
 *  Pi, S       device float d x d (the ones the corpus was quantised with)
 *  centroids   device float, 2^key_bits entries
 *  k           1..32 (and <= n_db)
 *  top_idx     device int64 [n_queries][k], top_scores device float [n_queries][k]
 *              (ids are row numbers of `db`; pass db rows [a, b) of a larger
 *              corpus and merge with tq_search_merge_topk, offset a)
 *  workspace   device scratch, 256-B aligned; queries run in blocks of as
 *              many as it holds (tq_search_workspace_bytes reports the size of
 *              one pass of up to 16,384 queries; any size from one query's
 *              share up works, a smaller one takes more passes)
 * Errors: TQ_ERR_INVALID_ARG, TQ_ERR_WORKSPACE (smaller than one query's
 * share), TQ_ERR_UNSUPPORTED (d not 64, 128 or 200), TQ_ERR_CUDA.
 * ---------------------------------------------------------------------- */
tq_status tq_search_topk(const tq_layout* layout, const void* q, tq_dtype q_dtype, int32_t n_queries,
                         const tq_planes* db, int64_t n_db, const float* Pi, const float* S,
                         const float* centroids, int32_t k, int64_t* top_idx, float* top_scores,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * tq_search_merge_topk — merge two per-query top-k lists (device), for a
 * corpus searched in shards (row ranges, several calls or several GPUs).
 *
 * Same ranking as tq_search_topk (decreasing score, equal scores by
 * increasing id). List X's ids are shifted by offset_x (the first corpus row
 * of its shard); id -1 marks an empty slot and never enters. Both inputs are
 * [n_queries][k], sorted as tq_search_topk writes them; the output, also
 * [n_queries][k], may alias either input.
 * Errors: TQ_ERR_INVALID_ARG (k outside 1..32, NULL, negative offsets), TQ_ERR_CUDA.
 * ---------------------------------------------------------------------- */
tq_status tq_search_merge_topk(int32_t n_queries, int32_t k,
                               const int64_t* idx_a, const float* scores_a, int64_t offset_a,
                               const int64_t* idx_b, const float* scores_b, int64_t offset_b,
                               int64_t* idx_out, float* scores_out, void* stream);

/* Scratch bytes tq_search_topk needs for one pass over min(n_queries, 16384)
 * queries (0 on invalid arguments). */
size_t tq_search_workspace_bytes(const tq_layout* layout, int32_t n_queries, int64_t n_db, int32_t k);

/* ------------------------------------------------------------------------
 * tq_fit_rotation — per-head rotation from calibration vectors (host only).
 *
 * gist.science TurboESM section 2B: instead of one global or random matrix,
 * a Pi is computed for every layer and attention head by SVD of real
 * activations, equalising the variance across directions.
 *
 *   X        host float [n][d]: the head's calibration vectors (uncentred)
 *   Pi_rand  host float [d][d]: the seeded random rotation
 *   Pi_out   host float [d][d]: Pi_rand V^T, V the right singular vectors of
 *            X (decreasing singular value; each signed so its largest-magnitude
 *            entry is positive)
 * Computed in fp64 (cyclic Jacobi on X^T X). Errors: TQ_ERR_INVALID_ARG.
 * ---------------------------------------------------------------------- */
tq_status tq_fit_rotation(int32_t d, const float* X, int64_t n, const float* Pi_rand, float* Pi_out);

/* ------------------------------------------------------------------------
 * tq_rotate_normalize — samples for the dual (K / V) codebooks (host only).
 *
 * gist.science TurboESM section 2C: K and V tables are fitted to their own
 * post-rotation coordinate distributions. Writes the coordinates of
 * Pi x / ||x|| for every non-zero row x of X (rows in order; zero rows have no
 * direction and are skipped) to u_out [n_out][d], fp64 internally.
 * Feed the pooled samples to tq_make_codebook(mode = 1).
 * ---------------------------------------------------------------------- */
tq_status tq_rotate_normalize(int32_t d, const float* X, int64_t n, const float* Pi, float* u_out, int64_t* n_out);

/* Description of the last error on this host thread ("" if none). */
const char* tq_last_error_string(void);

/* Library version string. */
const char* tq_version(void);

/* ------------------------------------------------------------------------
 * tq_kernel_launches — diagnostic, no counterpart in the pages.
 *
 * Number of kernels this library has launched (or recorded into a CUDA graph
 * under stream capture) since it was loaded, summed over all host threads and
 * devices. Library-internal memsets are not counted. Callers take the
 * difference of two readings around a region.
 * ---------------------------------------------------------------------- */
uint64_t tq_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
