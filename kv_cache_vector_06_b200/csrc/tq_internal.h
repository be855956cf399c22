// Internal declarations shared by the libtq translation units (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "tq.h"

#define TQ_MAX_LEVELS 16

// Read-only constants of one quantizer, passed to kernels by value (kernel parameter space).
struct TqConsts {
  int d;          // vector length (power of two, 8..1024)
  int bits;       // MSE bits per coordinate (1..4)
  int levels;     // 2^bits
  int m;          // QJL rows (0 or multiple of 32)
  int code_words; // 32-bit words per packed code row
  int sign_words; // 32-bit words per packed sign row
  int layout;     // tq_layout of the packed codes
  int fast_ok;    // codebook is an exact odd bit-plane expansion (tensor-core attention path)
  float plane_coef[4];   // e_P of c(code) = sum e_P s_P (+ e_3 s_0 s_1 s_2), s_P = 2 bit_P - 1
  float plane_coef_sum;  // sum of plane_coef
  float plane_coef_max;  // largest plane_coef
  float inv_sqrt_d;
  float qjl_scale;  // sqrt(pi/2)/m, 0 when m == 0
  float centroids[TQ_MAX_LEVELS];
  float thresholds[TQ_MAX_LEVELS];  // [levels-1] used
  const float *signs;  // device [d], +-1.0f (rotation D)
  const float *S;      // device [m][d] row-major (JL matrix)
  const float *St;     // device [d][m]: S transposed (coalesced reads with lane = row of S)
  int srht;               // S = P H D2 (structured QJL): encode transforms the residual instead
  const float *qjl_signs; // device [d], +-1.0f (D2), srht only
  int norm16;             // norm and rnorm stored as fp16 (else fp32)
  int polar;              // PolarQuant first stage (angle codes in place of coordinate codes)
  const float *polar_tab; // device [levels][thresholds | cos c | sin c][16], polar only
};

struct tq_ctx {
  int device;
  tq_spec spec;
  int64_t code_bytes;
  int64_t sign_bytes;
  double centroids[TQ_MAX_LEVELS];
  double thresholds[TQ_MAX_LEVELS];
  double mse_per_coord;
  float *dev_signs;  // [d]
  float *dev_S;      // [m][d]
  float *dev_St;     // [d][m]
  float *dev_qjl_signs;  // [d] (structured QJL only)
  float *dev_polar;      // PolarQuant angle tables (polar only)
  TqConsts k;        // kernel view
};

// ---------------------------------------------------------------- host helpers (api.cu)
tq_status tq_fail(tq_status st, const char *fmt, ...);
tq_status tq_cuda_check(cudaError_t e, const char *what);
// Makes a device current for the duration of one C-ABI call and restores the caller's
// current device when the call returns (the work itself is only enqueued).
class DeviceScope {
 public:
  DeviceScope() = default;
  DeviceScope(const DeviceScope &) = delete;
  DeviceScope &operator=(const DeviceScope &) = delete;
  ~DeviceScope() {
    if (prev_ >= 0) cudaSetDevice(prev_);
  }
  tq_status enter(int device) {
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return tq_cuda_check(e, "cudaGetDevice");
    if (cur == device) return TQ_OK;
    e = cudaSetDevice(device);
    if (e != cudaSuccess) return tq_cuda_check(e, "cudaSetDevice");
    prev_ = cur;
    return TQ_OK;
  }

 private:
  int prev_ = -1;
};

// ---------------------------------------------------------------- profile.cu
enum TqKernelKind {
  TQK_ROTATE_ENCODE = 0, TQK_QJL_PROJECT, TQK_ROTATE_QUERY, TQK_QUERY_PROJECT, TQK_SCORES,
  TQK_ATTEND_SPLIT, TQK_ATTEND_COMBINE, TQK_SEARCH_SCAN, TQK_SEARCH_MERGE, TQK_ATTEND_FRAG, TQK_DECODE_PREP,
  TQK_ENCODE_ROWS, TQK_ENCODE_QJL_TC, TQK_COUNT
};
bool tq_prof_on();  // per-kernel event profiling is enabled
void tq_prof_begin(int kind, cudaStream_t st);
void tq_prof_end(int kind, cudaStream_t st);

// ---------------------------------------------------------------- codebook.cpp
tq_status tq_codebook_fp64(int d, int bits, double *centroids, double *thresholds, double *mse);
// PolarQuant angle codebook of one level (level 1 uniform on (-pi, pi], levels >= 2 Lloyd-Max).
tq_status tq_polar_codebook_fp64(int level, int bits, double *centroids, double *thresholds);

// ---------------------------------------------------------------- kernels (launchers)
// Rotate rows of x: ENCODE mode normalises, quantizes, packs codes, writes norm (and, when the
// context has a QJL stage, the residual rows to `resid` and rnorm).  QUERY mode writes
// q' = (1/sqrt d) H D q (no normalisation) to `resid` as fp32 [n][d].
enum RotateMode { ROT_ENCODE = 0, ROT_QUERY = 1 };
// With `fsigns` set (d >= 128, QJL context), the projection and sign packing run in the same
// kernel (one vector per warp, S read from global memory): used for small batches such as the
// per-step append; large batches use the tiled projection kernel.
cudaError_t launch_rotate(const TqConsts &c, RotateMode mode, const void *x, tq_dtype dtype,
                          int64_t n, int64_t ld, const int64_t *slots, int64_t capacity,
                          uint32_t *codes, void *norm, void *rnorm, float *resid,
                          cudaStream_t st, uint32_t *fsigns = nullptr);
constexpr int64_t kFusedEncodeMaxRows = 4096;
// Bulk encode at d = 128, one row per thread (encode_tpr.cu): MSE-only contexts in either layout
// (token blocks: slots == NULL, whole blocks), structured-QJL contexts, and dense Gaussian QJL
// with m = d on bf16 rows (the projection on tcgen05).
bool encode_tpr_eligible(const TqConsts &c, const int64_t *slots, tq_dtype dtype);
int64_t encode_tpr_rows(const TqConsts &c, int64_t n);  // rows it takes (a block-layout tail is left)
cudaError_t launch_encode_tpr(const TqConsts &c, const void *x, tq_dtype dtype, int64_t n, int64_t ld,
                              const int64_t *slots, int64_t capacity, uint32_t *codes, void *norm, void *rnorm,
                              uint32_t *signs, cudaStream_t st);

// Z = R S^T for rows of R ([n][d] fp32).  SIGNS: pack bit = [z >= 0] into `signs` at the rows'
// slots.  DENSE: write Z as fp32 [n][m] to `zout`.
enum ProjEpilogue { PROJ_SIGNS = 0, PROJ_DENSE = 1 };
cudaError_t launch_project(const TqConsts &c, ProjEpilogue ep, const float *R, int64_t n,
                           const int64_t *slots, int64_t capacity, uint32_t *signs, float *zout,
                           cudaStream_t st);

// PolarQuant first stage at d = 128 (polar.cu): encode (codes, norm; with a QJL stage also the
// residual rows to `resid` and rnorm, for launch_project) and estimated scores.
bool polar_supported(const TqConsts &c);
cudaError_t launch_encode_polar(const TqConsts &c, const void *x, tq_dtype dtype, int64_t n, int64_t ld,
                                const int64_t *slots, int64_t capacity, uint32_t *codes, void *norm, void *rnorm,
                                float *resid, cudaStream_t st);
cudaError_t launch_scores_polar(const TqConsts &c, const float *qr, const float *p, int nq, const tq_packed &keys,
                                int64_t n, float *out, cudaStream_t st);

// out[i][k] = estimated score of prepared query i against slot k.
cudaError_t launch_scores(const TqConsts &c, const float *qr, const float *p, int nq,
                          const tq_packed &keys, int64_t n, float *out, cudaStream_t st);

// Attention over the compressed cache, split over the context, then combined.
struct AttnPlan {
  int group;        // n_q_heads / n_kv_heads
  int chunk;        // tokens per split
  int splits;       // splits per (batch, kv head)
  bool fast;        // tensor-core path (attend_mma.cu)
  bool fused;       // tensor-core path merges the splits itself (no combine launch)
  size_t extra;     // workspace bytes of the tensor-core path's query fragments and counters
};
AttnPlan attn_plan(const tq_attn_desc &desc, const TqConsts &kc, const TqConsts &vc);
size_t attn_partials_bytes(const tq_attn_desc &desc, const AttnPlan &plan, int d);
cudaError_t launch_attend(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc,
                          const AttnPlan &plan, const void *q, int dtype, const float *qr, const float *p,
                          float *partials, float *out, cudaStream_t st);
// attend_mma.cu
bool attn_fast_eligible(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc);
int attn_fast_chunk(const tq_attn_desc &desc);
constexpr int kFusedMaxSplits = 1024;
// the other translation units' shares of tq_device_status
cudaError_t rotate_device_flags(int *v, bool clear);
cudaError_t search_mma_device_flags(int *v, bool clear);
cudaError_t search_tc_device_flags(int *v, bool clear);
// Raise `func`'s dynamic shared-memory limit to at least `bytes` on the current device.  The
// attribute call is made once per (kernel, device) and larger size (it costs host time that would
// otherwise land between a kernel's launch and the work queued before it).
cudaError_t tq_smem_limit(const void *func, int bytes);  // splits merged inside the tensor-core kernel at most
size_t attn_fast_extra_bytes(const TqConsts &kc, const tq_attn_desc &desc);
cudaError_t launch_attend_fast(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc,
                               const AttnPlan &plan, const void *q, int dtype, void *extra,
                               float *partials, float *out, cudaStream_t st);
// Fused decode step (tensor-core path): append-encode nnew K and V rows at `slots`, build the
// query fragments, run the split kernel (which merges the splits when plan.fused; otherwise the
// caller then launches the combine).
cudaError_t launch_decode_step_fast(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc,
                                    const AttnPlan &plan, const void *knew, const void *vnew, int kvdtype,
                                    int64_t nnew, const int64_t *slots, const void *q, int qdtype, void *extra,
                                    float *partials, float *out, cudaStream_t st);
cudaError_t launch_attend_combine(const TqConsts &vc, const tq_attn_desc &desc, const AttnPlan &plan,
                                  const float *partials, float *out, cudaStream_t st);

// Search: per-(query tile, shard) top-k candidates, then a per-query merge.
struct SearchPlan {
  int qtile;   // queries per CTA
  int shards;  // row shards
};
SearchPlan search_plan(int nq, int64_t n, int k);
// Tensor-core scan (search_mma.cu): eligibility, workspace for the query fragments, shard count,
// and the scan (the existing merge then reduces the candidates).
// (the scan also needs norm and rnorm 16-byte aligned, and at most kSearchMmaMaxQ queries: 8 per
// grid row, 65535 rows)
constexpr int kSearchMmaMaxQ = 8 * 65535;
bool search_mma_eligible(const TqConsts &c);
// tcgen05 scan (search_tc.cu): 64 queries per CTA, k <= 16, at least 32 queries
bool search_tc_eligible(const TqConsts &c, int nq, int k);
size_t search_tc_ws_bytes(const TqConsts &c, int nq);
int search_tc_shards(int nq, int64_t n);
cudaError_t launch_search_tc(const TqConsts &c, int shards, const float *qr, const float *p, int nq,
                             const tq_packed &db, int64_t n, int k, void *ws, float *cand_s, int64_t *cand_i,
                             cudaStream_t st);
size_t search_mma_frag_bytes(const TqConsts &c, int nq);
int search_mma_shards(const TqConsts &c, int nq, int64_t n, int k);
cudaError_t launch_search_mma(const TqConsts &c, int shards, const float *qr, const float *p, int nq,
                              const tq_packed &db, int64_t n, int k, void *fragws, float *cand_s, int64_t *cand_i,
                              cudaStream_t st);
cudaError_t launch_search_merge(int nq, int shards, int k, const float *cand_s, const int64_t *cand_i, float *out_s,
                                int64_t *out_i, cudaStream_t st);
// Large k (32 < k <= 1024): CUDA-core scan with per-query shared-memory top-k buffers, then a
// merge of the shards' lists in the same way (search.cu).
constexpr int kSearchMaxK = 1024;
constexpr int kSearchWarpMaxK = 32;  // above this, the large-k scan
int search_bigk_shards(int nq, int64_t n);
cudaError_t launch_search_bigk(const TqConsts &c, int shards, const float *qr, const float *p, int nq,
                               const tq_packed &db, int64_t n, int k, float *cand_s, int64_t *cand_i,
                               float *out_s, int64_t *out_i, cudaStream_t st);
cudaError_t launch_search(const TqConsts &c, const SearchPlan &plan, const float *qr,
                          const float *p, int nq, const tq_packed &db, int64_t n, int k,
                          float *cand_s, int64_t *cand_i, float *out_s, int64_t *out_i,
                          cudaStream_t st);

static inline int64_t tq_align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }
// SMs of the current device (148 on a B200 if the query fails).
static inline int tq_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
      n > 0)
    return n;
  return 148;
}
