// tq_search_topk: inner-product top-k over a packed database ("谷歌 TurboQuant 深度拆解"
// 第三部分 "向量搜索"), ordered by (estimated score descending, index ascending).
//
// Scan: a CTA takes a tile of 8 queries and one shard of rows.  For each block of 256 rows every
// thread scores one row against the 8 prepared queries (shared memory, broadcast reads) into a
// shared tile; then warp w merges query w's 256 scores into its running top-k, which lives one
// entry per lane (k <= 32) and is updated by ballot + shuffle insertion.  Each CTA writes its
// shard's candidates; a merge kernel (one warp per query) reduces the shards to the final list.
#include <cmath>

#include "device_common.cuh"

namespace {

constexpr int kSrThreads = 256;
constexpr int kSrQ = 8;  // queries per CTA = warps per CTA

__global__ void __launch_bounds__(kSrThreads)
search_scan_kernel(TqConsts c, const float *__restrict__ qr, const float *__restrict__ p, int nq,
                   tq_packed db, int64_t n, int k, int64_t rows_per_shard, int shards,
                   float *__restrict__ cand_s, int64_t *__restrict__ cand_i) {
  extern __shared__ float sm[];
  float *qs = sm;                       // [d][8]
  float *ps = qs + c.d * kSrQ;          // [m][8]
  float *cent = ps + c.m * kSrQ;        // [16]
  float *tile = cent + TQ_MAX_LEVELS;   // [8][256]
  const int shard = blockIdx.x;
  const int q0 = blockIdx.y * kSrQ;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < c.d * kSrQ; i += kSrThreads) {
    const int j = i / kSrQ, q = i % kSrQ;
    qs[i] = (q0 + q < nq) ? qr[(int64_t)(q0 + q) * c.d + j] : 0.f;
  }
  for (int i = tid; i < c.m * kSrQ; i += kSrThreads) {
    const int j = i / kSrQ, q = i % kSrQ;
    ps[i] = (q0 + q < nq) ? p[(int64_t)(q0 + q) * c.m + j] : 0.f;
  }
  if (tid < TQ_MAX_LEVELS) cent[tid] = c.centroids[tid];
  __syncthreads();

  const int64_t r_begin = (int64_t)shard * rows_per_shard;
  const int64_t r_end = min(n, r_begin + rows_per_shard);
  float bs = -INFINITY;
  int64_t bi = INT64_MAX;
  const uint32_t *codes = static_cast<const uint32_t *>(db.codes);
  const uint32_t *signs = static_cast<const uint32_t *>(db.signs);
  for (int64_t r0 = r_begin; r0 < r_end; r0 += kSrThreads) {
    const int64_t row = r0 + tid;
    float sc[kSrQ];
    if (row < r_end) {
      estimate_scores<kSrQ>(c, codes + row * c.code_words,
                            c.m > 0 ? signs + row * c.sign_words : nullptr, db.norm[row],
                            c.m > 0 ? db.rnorm[row] : 0.f, qs, ps, cent, sc);
    } else {
#pragma unroll
      for (int q = 0; q < kSrQ; ++q) sc[q] = -INFINITY;
    }
#pragma unroll
    for (int q = 0; q < kSrQ; ++q) tile[q * kSrThreads + tid] = sc[q];
    __syncthreads();
    if (q0 + warp < nq) {
#pragma unroll
      for (int cchunk = 0; cchunk < kSrThreads / 32; ++cchunk) {
        const int idx = cchunk * 32 + lane;
        const int64_t rr = r0 + idx;
        warp_topk_insert(bs, bi, k, tile[warp * kSrThreads + idx], rr, rr < r_end);
      }
    }
    __syncthreads();
  }
  if (q0 + warp < nq && lane < k) {
    const int64_t o = ((int64_t)(q0 + warp) * shards + shard) * k + lane;
    cand_s[o] = bs;
    cand_i[o] = bi;
  }
}

__global__ void search_merge_kernel(int nq, int shards, int k, const float *__restrict__ cand_s,
                                    const int64_t *__restrict__ cand_i, float *__restrict__ out_s,
                                    int64_t *__restrict__ out_i) {
  const int q = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (q >= nq) return;
  float bs = -INFINITY;
  int64_t bi = INT64_MAX;
  const int64_t total = (int64_t)shards * k;
  const float *cs = cand_s + (int64_t)q * total;
  const int64_t *ci = cand_i + (int64_t)q * total;
  for (int64_t c0 = 0; c0 < total; c0 += 32) {
    const int64_t o = c0 + lane;
    const bool v = o < total && ci[o] != INT64_MAX;
    warp_topk_insert(bs, bi, k, v ? cs[o] : -INFINITY, v ? ci[o] : INT64_MAX, v);
  }
  if (lane < k) {
    out_s[(int64_t)q * k + lane] = bs;
    out_i[(int64_t)q * k + lane] = bi;
  }
}

}  // namespace

SearchPlan search_plan(int nq, int64_t n, int k) {
  (void)k;
  SearchPlan p;
  p.qtile = kSrQ;
  const int64_t qtiles = (nq + kSrQ - 1) / kSrQ;
  int64_t shards = qtiles > 0 ? (4 * 148 + qtiles - 1) / qtiles : 1;
  const int64_t max_shards = (n + kSrThreads - 1) / kSrThreads;
  if (shards > max_shards) shards = max_shards;
  if (shards < 1) shards = 1;
  p.shards = (int)shards;
  return p;
}

cudaError_t launch_search(const TqConsts &c, const SearchPlan &plan, const float *qr,
                          const float *p, int nq, const tq_packed &db, int64_t n, int k,
                          float *cand_s, int64_t *cand_i, float *out_s, int64_t *out_i,
                          cudaStream_t st) {
  if (nq <= 0) return cudaSuccess;
  const int64_t rows_per_shard = (n + plan.shards - 1) / plan.shards;
  const size_t smem = sizeof(float) * ((size_t)(c.d + c.m) * kSrQ + TQ_MAX_LEVELS + kSrQ * kSrThreads);
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(search_scan_kernel), (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)plan.shards, (unsigned)((nq + kSrQ - 1) / kSrQ));
  tq_prof_begin(TQK_SEARCH_SCAN, st);
  search_scan_kernel<<<grid, kSrThreads, smem, st>>>(c, qr, p, nq, db, n, k, rows_per_shard, plan.shards,
                                                     cand_s, cand_i);
  tq_prof_end(TQK_SEARCH_SCAN, st);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_search_merge(nq, plan.shards, k, cand_s, cand_i, out_s, out_i, st);
}

cudaError_t launch_search_merge(int nq, int shards, int k, const float *cand_s, const int64_t *cand_i, float *out_s,
                                int64_t *out_i, cudaStream_t st) {
  const int wpb = 4;
  tq_prof_begin(TQK_SEARCH_MERGE, st);
  search_merge_kernel<<<(unsigned)((nq + wpb - 1) / wpb), 32 * wpb, 0, st>>>(nq, shards, k, cand_s, cand_i, out_s,
                                                                             out_i);
  tq_prof_end(TQK_SEARCH_MERGE, st);
  return cudaGetLastError();
}
