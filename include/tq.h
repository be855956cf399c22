/*
 * tq.h — C ABI of libtq, a B200 (sm_100a) implementation of the TurboQuant hot path:
 * encode (random rotation, stored norm, Lloyd-Max codes, bit-packing, QJL sign sketch of the
 * residual), scoring of full-precision queries against packed keys, decode attention over a
 * compressed KV cache, and inner-product top-k search over a compressed database.
 *
 * Sources (web pages, by title and section):
 *   [LP] "TurboQuant 学习路径：论文 → 技术 → 数学" (zzszmyf.github.io)
 *   [JJ] "谷歌 TurboQuant 深度拆解：LLM 内存压缩 6 倍、推理加速 8 倍、零精度损失" (juejin.cn)
 *   [VC] vocus.cc article on TurboQuant (PolarQuant stage, QJL 1-bit stage)
 *   [ZC] "TurboQuant+ 深度解析" (zhichai.net)
 * The pages print no API ([JJ] 第四部分 "没有官方代码"); the calls below follow the problem the
 * pages state: compress key/value or database vectors with no per-block constants, then score a
 * full-precision query against the compressed keys ([JJ] 第一部分, 第二部分).
 *
 * Conventions for every call:
 *   - Plain C; no allocation on the data calls (encode, scores, attend, search); the caller owns
 *     every data buffer (inputs, packed arrays, outputs, workspace) and passes raw pointers.
 *   - "device" pointers are CUDA global-memory addresses on the context's device; "host"
 *     pointers are ordinary CPU memory.  Device buffers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Data calls
 *     only enqueue work and return; results are ready when the stream reaches that point.
 *   - Arguments are validated on the host before any launch: a bad shape, pointer or alignment
 *     returns TQ_EINVAL, an unsupported size TQ_EUNSUPPORTED, and nothing is launched.  A launch
 *     failure returns TQ_ECUDA.  tq_last_error() then holds a one-line, thread-local message.
 *   - Input values are not checked: NaN or Inf inputs give undefined outputs.
 *   - Kernels never trap or assert; out-of-range slots or block-table entries are skipped.
 *   - Outputs are undefined after an error.
 *
 * Supported sizes: d (vector length) a power of two in [8, 1024]; mse_bits in [1, 4];
 * qjl_m = 0 (MSE stage only) or a multiple of 32 in [32, 1024]; attention group size
 * n_q_heads / n_kv_heads in {1, 2, 4, 8}; search k in [1, 1024].
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
  TQ_EINVAL = 1,        /* bad argument: null pointer, bad shape, misaligned buffer, ws too small */
  TQ_EUNSUPPORTED = 2,  /* well-formed but outside the supported sizes listed above */
  TQ_ENOMEM = 3,        /* context creation could not allocate its constants */
  TQ_ECUDA = 4,         /* a CUDA call or kernel launch failed */
  TQ_ETIMEOUT = 5       /* a kernel gave up a bounded wait for its own asynchronous copies; returned
                           by tq_device_status, which reports it (see TQ_DEVFLAG_STAGING_TIMEOUT) */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

/* Quantizer shape for one tensor role (keys, values, or a search database).
 *   d        vector length
 *   mse_bits b: bits per coordinate of the Lloyd-Max stage (2^b levels)
 *   qjl_m    m: rows of the Gaussian JL matrix S (1 sign bit each); 0 = no QJL stage
 * "b bits per coordinate" for keys in the pages' sense = (b-1) MSE bits + 1 QJL bit with m = d
 * ([JJ] 第二部分 "两步结合的效果": 2 + 1 = 3 bits). */
typedef struct {
  int32_t d;
  int32_t mse_bits;
  int32_t qjl_m;
  int32_t layout;     /* tq_layout of the packed codes (TQ_LAYOUT_ROWS unless stated) */
  int32_t norm_bits;  /* storage of norm and rnorm: 32 (or 0) = fp32, 16 = fp16 (IEEE half, round
                         to nearest, values above 65504 stored as 65504).  The norms are the only
                         per-vector constants, and quantizers keep such constants in FP16 or FP32
                         ([JJ] 第一部分); fp16 saves 4 bytes per vector with a QJL stage, 0.25 bit
                         per coordinate at d = 128. */
} tq_spec;

/* Packed-code layouts.
 *   TQ_LAYOUT_ROWS     every slot owns one code row (see tq_packed).
 *   TQ_LAYOUT_BLOCK16  token-transposed blocks for attention values: MSE-only contexts
 *                      (qjl_m == 0), capacities a multiple of 16.  Slots 16k .. 16k+15 share the
 *                      16 * code_bytes bytes of block k, read as little-endian 32-bit words W:
 *                        W[q*d + j], q < b/2:  bit t      = bit 2q   of code_j of slot 16k+t,
 *                                              bit 16 + t = bit 2q+1 of code_j of slot 16k+t;
 *                        W[(b/2)*d + j/2] (b odd): bit 16*(j%2) + t = bit b-1 of code_j of slot 16k+t,
 *                      for t in [0,16), j in [0,d).  One word then holds one coordinate of 16
 *                      tokens in two planes, the operand shape of the tensor-core value sum. */
typedef enum { TQ_LAYOUT_ROWS = 0, TQ_LAYOUT_BLOCK16 = 1 } tq_layout;

/* Packed, caller-owned device arrays indexed by slot (one slot = one encoded vector).
 *   codes  [capacity][code_bytes]  b bit-planes of d bits, plane t holding bit t of every code:
 *                                  bit t of code_j is bit (t*d + j) of the vector's
 *                                  little-endian bit stream; padded to a multiple of 16 bytes.
 *   signs  [capacity][sign_bytes]  QJL bits, bit i = [ (S r)_i >= 0 ]; NULL when qjl_m == 0.
 *   norm   [capacity]  ||x||, fp32 or fp16 per tq_spec.norm_bits (4- or 2-byte aligned)
 *   rnorm  [capacity]  ||r||, r the rotated-domain residual, same type; NULL when qjl_m == 0.
 * code_bytes = roundup(b*d/8, 16), sign_bytes = roundup(m/8, 16) (tq_ctx_layout).  The
 * tensor-core attention path also wants the norm arrays 16-byte aligned (it copies them in bulk);
 * other alignments take the general path. */
typedef struct {
  void *codes;
  void *signs;
  void *norm;
  void *rnorm;
  int64_t capacity;
} tq_packed;

typedef struct tq_ctx tq_ctx; /* opaque; owns read-only device constants, usable from any stream */

/* Decode-attention descriptor.  Query head hq of sequence b reads KV head hq / (n_q_heads /
 * n_kv_heads) over tokens [0, seq_lens[b]).  The slot of token t is
 *   contiguous (block_table == NULL): (b * n_kv_heads + h) * ctx_stride + t
 *   paged:      (block_table[b * max_blocks + t / block_size] * n_kv_heads + h) * block_size
 *               + t % block_size
 * in both the K and the V packed arrays. */
typedef struct {
  int32_t batch;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  float scale;                 /* softmax scale on the estimated scores; 0 = 1/sqrt(d) */
  const int32_t *seq_lens;     /* device [batch]; values above max_seq_len are clamped to it */
  const int32_t *block_table;  /* device [batch][max_blocks] or NULL (contiguous) */
  int32_t max_blocks;          /* row stride of block_table */
  int32_t block_size;          /* tokens per block (paged); ignored when contiguous */
  int64_t ctx_stride;          /* slots per (batch, kv head) row (contiguous); ignored when paged */
  int32_t max_seq_len;         /* host-known upper bound of seq_lens; sizes the split grid */
  tq_packed k;                 /* keys, encoded with the K context */
  tq_packed v;                 /* values, encoded with the V context (MSE stage only) */
  float sparse_v;              /* Sparse V threshold tau ("TurboQuant+ 深度解析" 第六部分): value rows
                                  whose softmax weight is below tau are not dequantized; 0 = off.
                                  Tensor-core path (TQ_LAYOUT_BLOCK16 values): a row is dropped
                                  when a running bound on its weight is below tau, so every dropped
                                  row has final weight < tau; the general path ignores it. */
} tq_attn_desc;

/* Lloyd-Max codebook for one coordinate of a randomly rotated unit vector in R^d.
 * [JJ] 第六部分 "为什么随机旋转这么关键" gives the coordinate density
 *   f_X(x) = Gamma(d/2)/(sqrt(pi) Gamma((d-1)/2)) (1-x^2)^((d-3)/2) on [-1, 1];
 * [JJ] 第二部分 第一步 and [LP] 三.4 name the Lloyd-Max quantizer for it.  Host-only, fp64.
 *   centroids     host out [2^bits], ascending
 *   thresholds    host out [2^bits - 1], midpoints of neighbouring centroids
 *   mse_per_coord host out, nullable: E[(X - Q(X))^2]
 * Errors: TQ_EINVAL on null outputs; TQ_EUNSUPPORTED outside the supported d and bits. */
tq_status tq_make_codebook(int32_t d, int32_t bits, double *centroids, double *thresholds,
                           double *mse_per_coord);

/* Create a quantizer context on `device`: builds the codebook and uploads the rotation signs D,
 * the JL matrix S and the codebook (fp32) once.  D and S are drawn by the caller
 * ([LP] 二.2: FJLT D = random signs; standard JL R_ij ~ N(0,1)); the same D and S must be used
 * to encode and to score.
 *   spec        host, read during the call
 *   rot_signs   host int8 [d], entries +1 or -1
 *   qjl_matrix  host fp32 [qjl_m][d] row-major; may be NULL when qjl_m == 0
 *   out         host out: the new context
 * Errors: TQ_EINVAL (nulls, a sign not +-1), TQ_EUNSUPPORTED (sizes), TQ_ENOMEM, TQ_ECUDA. */
tq_status tq_ctx_create(const tq_spec *spec, const int8_t *rot_signs, const float *qjl_matrix,
                        int32_t device, tq_ctx **out);

/* Create a context whose QJL stage uses a structured JL matrix instead of a caller-drawn dense
 * Gaussian one ([LP] 二.2 "Johnson-Lindenstrauss 实现技术": the fast JL transform y = P H D x):
 *   S = P H D2,  S[i][j] = H[i][j] D2[j] for i < qjl_m,
 * H the d x d Sylvester Hadamard matrix left unnormalised (entries +-1), D2 a diagonal of random
 * signs drawn independently of the rotation's, P keeping the first qjl_m rows.  The entries are
 * +-1 with unit variance like N(0,1) draws, the rows are orthogonal, and the estimator keeps the
 * sqrt(pi/2)/m scale; over D2 it is unbiased to within Monte-Carlo resolution (exactly so only for
 * Gaussian rows).  Encode computes S r as a Walsh-Hadamard transform of D2 r in registers: no
 * projection matrix is read and tq_encode_workspace_size is 0.  Every other call is unchanged.
 *   spec        host; qjl_m a multiple of 32 in [32, d]
 *   rot_signs   host int8 [d], entries +1 or -1 (D)
 *   qjl_signs   host int8 [d], entries +1 or -1 (D2)
 *   out         host out: the new context
 * Errors: TQ_EINVAL (nulls, a sign not +-1), TQ_EUNSUPPORTED (sizes, qjl_m = 0 or > d),
 * TQ_ENOMEM, TQ_ECUDA. */
tq_status tq_ctx_create_srht(const tq_spec *spec, const int8_t *rot_signs, const int8_t *qjl_signs,
                             int32_t device, tq_ctx **out);

/* Create a context whose first stage is PolarQuant instead of the per-coordinate quantizer
 * ([JJ] 第二部分 第一步 "PolarQuant——换一个坐标系来看数据"; [VC] 第一階段): after the same random
 * rotation, coordinates are paired into (radius, angle), the radii paired again, recursively, to
 * one radius (the stored norm) and d - 1 angles, each angle quantized with spec->mse_bits bits by
 * the Lloyd-Max codebook of its level's known law (tq_polar_codebook); no per-block constants.
 * The QJL stage, when qjl_m > 0, sketches the residual y/||x|| - y^ with the dense S as usual.
 * Packed arrays as for tq_ctx_create: code slot p holds angle p (level 1 first: d/2 angles, then
 * level 2, ..., the last level's single angle at d - 2; slot d - 1 is 0).  Every call accepts such
 * contexts (for keys, values or a database): scores through the reconstructed direction y^, value
 * coordinates as products of the cos / sin of the angles along their path.  They take the CUDA-core
 * attention and search paths (the tensor-core paths rest on the coordinate codebook's bit planes).
 *   spec  d = 128, TQ_LAYOUT_ROWS, mse_bits 1..4, qjl_m 0 or a multiple of 32 up to 1024
 * Errors: as tq_ctx_create; TQ_EUNSUPPORTED for other d or layouts. */
tq_status tq_ctx_create_polar(const tq_spec *spec, const int8_t *rot_signs, const float *qjl_matrix,
                              int32_t device, tq_ctx **out);

/* PolarQuant angle codebook of one level (host, fp64).  Level 1 angles of a uniformly random
 * direction are uniform on (-pi, pi]: 2^bits equal cells from -pi, centroids at the cell middles.
 * A level-l angle, l >= 2, is atan2 of two independent radii of k = 2^(l-1) coordinates each, with
 * density 2 (sin a cos a)^(k-1) / B(k/2, k/2) on [0, pi/2]: its Lloyd-Max codebook.
 *   centroids host out [2^bits], thresholds host out [2^bits - 1]
 * Errors: TQ_EINVAL (nulls), TQ_EUNSUPPORTED (level outside 1..10, bits outside 1..4). */
tq_status tq_polar_codebook(int32_t level, int32_t bits, double *centroids, double *thresholds);

/* Free a context (NULL is accepted).  The caller must ensure no queued work still uses it. */
tq_status tq_ctx_destroy(tq_ctx *ctx);

/* Bytes per slot of the packed code and sign arrays for this context (host out pointers). */
tq_status tq_ctx_layout(const tq_ctx *ctx, int64_t *code_bytes, int64_t *sign_bytes);

/* Encode n vectors into packed slots ([JJ] 第二部分 第一步 + 第二步; [VC] 第一/二階段):
 *   nu = ||x||, u = x/nu (0 if nu = 0), y = (1/sqrt(d)) H (D u),
 *   code_j = #{thresholds <= y_j}, r = y - c[code], gamma = ||r||, bit_i = [(S r)_i >= 0].
 *   x      device [n][ld] of dtype (row i at x + i*ld elements), ld >= d
 *   slots  device int64 [n] or NULL: row i goes to slot slots[i] (or i); rows whose slot is
 *          outside [0, out.capacity) are skipped
 *   out    packed arrays written at those slots
 *   ws     device workspace of tq_encode_workspace_size() bytes (NULL allowed when that is 0)
 * Errors: TQ_EINVAL (nulls, ld < d, n < 0, alignment, ws too small), TQ_ECUDA. */
tq_status tq_encode_workspace_size(const tq_ctx *ctx, int64_t n, size_t *bytes);
tq_status tq_encode_kv(const tq_ctx *ctx, const void *x, tq_dtype dtype, int64_t n, int64_t ld,
                       const int64_t *slots, tq_packed out, void *ws, size_t ws_bytes,
                       void *stream);

/* Estimated inner products of nq full-precision queries with n packed keys (slots 0..n-1);
 * the context must use TQ_LAYOUT_ROWS
 * ([JJ] 第二部分 第二步 and 第六部分 "无偏估计的数学保证"):
 *   q' = (1/sqrt(d)) H (D q), p = S q',
 *   out[i][k] = nu_k ( <q', c[code_k]> + sqrt(pi/2)/m * gamma_k * sum_j (2 bit_kj - 1) p_j ).
 *   q    device [nq][d] of dtype
 *   out  device fp32 [nq][n]
 *   ws   device workspace of tq_scores_workspace_size() bytes
 * Errors: TQ_EINVAL (nulls, n > keys.capacity, alignment, ws too small), TQ_ECUDA. */
tq_status tq_scores_workspace_size(const tq_ctx *ctx, int32_t nq, size_t *bytes);
tq_status tq_scores(const tq_ctx *ctx, const void *q, tq_dtype dtype, int32_t nq, tq_packed keys,
                    int64_t n, float *out, void *ws, size_t ws_bytes, void *stream);

/* One decode step of attention over the compressed cache ([JJ] 第一部分 "KV 缓存是什么",
 * 第三部分 "推理速度"): logits = scale * estimated scores against the K cache, softmax over the
 * sequence, output = sum_t w_t * nu_t * D_V (1/sqrt(d)) H c_V[code_t] (V's MSE stage).
 *   kctx, vctx  contexts used to encode K and V (same d; kctx in TQ_LAYOUT_ROWS; vctx with
 *               qjl_m == 0, either layout; TQ_LAYOUT_BLOCK16 values enable the tensor-core path)
 *   q           device [batch][n_q_heads][d] of dtype
 *   out         device fp32 [batch][n_q_heads][d]; an empty sequence gives zeros
 *   ws          device workspace of tq_attend_workspace_size() bytes
 * Errors: TQ_EINVAL (nulls, shapes, alignment, ws too small), TQ_EUNSUPPORTED (group size,
 * vctx with a QJL stage, d mismatch), TQ_ECUDA. */
tq_status tq_attend_workspace_size(const tq_ctx *kctx, const tq_ctx *vctx,
                                   const tq_attn_desc *desc, size_t *bytes);
tq_status tq_attend_decode(const tq_ctx *kctx, const tq_ctx *vctx, const tq_attn_desc *desc,
                           const void *q, tq_dtype dtype, float *out, void *ws, size_t ws_bytes,
                           void *stream);

/* One serving decode step: append the new token's key and value of every (sequence, KV head)
 * to the compressed cache, then attend with the new queries (tq_encode_kv for K and for V, then
 * tq_attend_decode, as one call).  With the tensor-core attention path the appends and the
 * query preparation run in a single launch.
 *   k_new, v_new  device [n_new][d] of kv_dtype, contiguous rows
 *   new_slots     device int64 [n_new]: slot of each new row in desc->k and desc->v
 *   desc          as for tq_attend_decode; desc->seq_lens must already count the new tokens
 *   q, out        as for tq_attend_decode
 *   ws            device workspace of tq_decode_step_workspace_size() bytes
 * Errors: as tq_encode_kv and tq_attend_decode; TQ_EINVAL if n_new > 4096. */
tq_status tq_decode_step_workspace_size(const tq_ctx *kctx, const tq_ctx *vctx, const tq_attn_desc *desc,
                                        int64_t n_new, size_t *bytes);
tq_status tq_decode_step(const tq_ctx *kctx, const tq_ctx *vctx, const tq_attn_desc *desc,
                         const void *k_new, const void *v_new, tq_dtype kv_dtype, int64_t n_new,
                         const int64_t *new_slots, const void *q, tq_dtype q_dtype, float *out,
                         void *ws, size_t ws_bytes, void *stream);

/* Allocation-free decode attention.  The pages have no counterpart: this entry point exists for
 * callers that cannot allocate device memory when they run attention, such as an inference
 * engine that gives all device memory to its own pool at start-up and forbids extensions from
 * calling cudaMalloc, or a latency-critical decode loop in which an allocator call could
 * synchronize the device.
 * Same arguments, layouts and results as tq_attend_decode, without the workspace: the scratch
 * space is one fixed TQ_NOALLOC_SCRATCH_BYTES (8 MiB) array of device memory that the library
 * defines statically; every GPU that loads the library keeps it until the process exits.
 *   - The first call on a device looks up that array's device address (cudaGetSymbolAddress,
 *     with the context's device made current) and caches it; make this first call before any
 *     CUDA graph capture on that device.
 *   - A request whose tq_attend_workspace_size exceeds TQ_NOALLOC_SCRATCH_BYTES returns
 *     TQ_EINVAL with a message naming both sizes; nothing is launched.
 *   - All calls on a device share the array and leave their contents in it.  No element needs to
 *     start at zero (each call writes what it reads), but calls that overlap on the GPU (other
 *     streams, other host threads) race on it: order them on one stream or with events.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine (with the tq_profile_*
 *     instrumentation switched on, the library creates CUDA event objects as for any call). */
#define TQ_NOALLOC_SCRATCH_BYTES (8u << 20)
tq_status tq_attend_decode_noalloc(const tq_ctx *kctx, const tq_ctx *vctx, const tq_attn_desc *desc,
                                   const void *q, tq_dtype dtype, float *out, void *stream);

/* Inner-product top-k over n packed database vectors (slots 0..n-1) ([JJ] 第三部分 "向量搜索");
 * the context must use TQ_LAYOUT_ROWS:
 * order by (estimated score descending, index ascending).
 *   q           device [nq][d] of dtype
 *   out_scores  device fp32 [nq][k]
 *   out_idx     device int64 [nq][k]
 *   ws          device workspace of tq_search_workspace_size() bytes (16-byte aligned; covers
 *               every scan the call may choose)
 * The scan depends on the shape. With k <= 32, d in {128, 256, 512, 1024} with qjl_m = d, 1-3
 * MSE bits and a symmetric codebook runs on tensor cores:
 *   - nq >= 32 and k <= 16: tcgen05 MMAs, 64 queries per CTA;
 *   - otherwise mma.sync, 8 queries per CTA (norm and rnorm 16-byte aligned);
 *   - any other shape with k <= 32, or unaligned norms for the second case: CUDA cores, 8 queries
 *     per CTA, one running top-k list per warp;
 *   - 32 < k <= 1024: CUDA cores, 4 queries per CTA, each query's running top-k kept in shared
 *     memory with the candidates that beat its current k-th entry, sorted (bitonic) when the
 *     buffer fills; the shards' lists are merged the same way.
 * All give the same top-k within the documented tolerances (the tensor-core scans round each
 * query term to 2^-23 of the query's largest term).
 * Errors: TQ_EINVAL (nulls, k < 1, k > n, alignment, ws too small), TQ_EUNSUPPORTED (k > 1024),
 * TQ_ECUDA.  A scan that gave up waiting for its copies sets TQ_DEVFLAG_STAGING_TIMEOUT (see
 * tq_device_status) and leaves its outputs unspecified. */
tq_status tq_search_workspace_size(const tq_ctx *ctx, int32_t nq, int64_t n, int32_t k,
                                   size_t *bytes);
tq_status tq_search_topk(const tq_ctx *ctx, const void *q, tq_dtype dtype, int32_t nq,
                         tq_packed db, int64_t n, int32_t k, float *out_scores, int64_t *out_idx,
                         void *ws, size_t ws_bytes, void *stream);

/* Instrumentation, off by default.  While enabled, every kernel that a data call launches is
 * bracketed by two CUDA events recorded on the caller's stream (so the pair times exactly that
 * kernel on the stream it runs on).  tq_profile_read waits for the recorded events and reports,
 * for kernel kind `index` (0, 1, ... until it returns TQ_EINVAL), its name, the number of
 * launches and their summed device time in milliseconds since the last reset.  Do not enable
 * while capturing a CUDA graph.  While enabled, the attention kernel is launched without
 * programmatic dependence on the kernel before it (an event sits between them).
 *   name  host out buffer of name_len bytes (nullable); launches, total_ms host outs (nullable) */
tq_status tq_profile_enable(int32_t on);
tq_status tq_profile_reset(void);
tq_status tq_profile_read(int32_t index, char *name, int32_t name_len, int64_t *launches,
                          double *total_ms);

/* Device-side status of the library on `device`: the TQ_DEVFLAG_* bits raised by kernels since
 * the last clear.  Synchronizes the device first; clear != 0 resets the bits.  Every wait of a
 * kernel for its own asynchronous copies (bulk copies on an mbarrier) is bounded: a kernel that
 * gives up (after about a second) raises TQ_DEVFLAG_STAGING_TIMEOUT, waits once more (bounded)
 * for the copies it issued, and returns without writing its outputs; the CUDA context stays
 * usable.  The caller's current device is restored on return.
 *   flags  host out (written whenever the device could be read, also with TQ_ETIMEOUT)
 * Returns TQ_ETIMEOUT when TQ_DEVFLAG_STAGING_TIMEOUT is among the flags read (the outputs of the
 * work since the last clear are then unspecified), else TQ_OK.
 * Errors: TQ_EINVAL (null flags), TQ_ECUDA. */
#define TQ_DEVFLAG_STAGING_TIMEOUT 1
tq_status tq_device_status(int32_t device, int32_t *flags, int32_t clear);

/* Test hook for the bounded waits, off by default; the pages have no counterpart.  With
 * polls > 0, every CTA of the tensor-core attention kernel on `device` first makes one bounded
 * wait of `polls` polls on a shared-memory barrier that is armed for bytes no copy sends, so the
 * wait runs out (no fault, no unbounded wait): the CTA raises TQ_DEVFLAG_STAGING_TIMEOUT, drains
 * the copies it had already issued, and returns.  polls = 0 switches the hook off.  Synchronous
 * with respect to the host; not for use while other work runs on the device.
 * Errors: TQ_EINVAL (polls < 0), TQ_ECUDA. */
tq_status tq_debug_wait_probe(int32_t device, int32_t polls);

/* Thread-local description of the last error on this thread ("" if none). */
const char *tq_last_error(void);

/* Library version string. */
const char *tq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
