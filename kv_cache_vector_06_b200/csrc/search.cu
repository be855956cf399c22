// tq_search_topk: inner-product top-k over a packed database ("谷歌 TurboQuant 深度拆解"
// 第三部分 "向量搜索"), ordered by (estimated score descending, index ascending).
//
// Scan: a CTA takes a tile of 8 queries and one shard of rows.  For each block of 256 rows every
// thread scores one row against the 8 prepared queries (shared memory, broadcast reads; PolarQuant
// rows through their reconstructed direction) into a shared tile; then warp w merges query w's 256 scores into its running top-k, which lives one
// entry per lane (k <= 32) and is updated by ballot + shuffle insertion.  Each CTA writes its
// shard's candidates; a merge kernel (one warp per query) reduces the shards to the final list.
#include <cmath>

#include "device_common.cuh"
#include "polar_device.cuh"

namespace {

constexpr int kSrThreads = 256;
constexpr int kSrQ = 8;  // queries per CTA = warps per CTA

template <bool POLAR>
__global__ void __launch_bounds__(kSrThreads)
search_scan_kernel(TqConsts c, const float *__restrict__ qr, const float *__restrict__ p, int nq,
                   tq_packed db, int64_t n, int k, int64_t rows_per_shard, int shards,
                   float *__restrict__ cand_s, int64_t *__restrict__ cand_i) {
  extern __shared__ float sm[];
  float *qs = sm;                       // [d][8]
  float *ps = qs + c.d * kSrQ;          // [m][8]
  float *cent = ps + c.m * kSrQ;        // [16]
  float *tile = cent + TQ_MAX_LEVELS;   // [8][256]
  __shared__ PolarTab ptab;              // PolarQuant contexts: the angle tables
  const int shard = blockIdx.x;
  const int q0 = blockIdx.y * kSrQ;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (POLAR) polar_tab_stage(ptab, c.polar_tab, tid, kSrThreads);
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
      const uint32_t *cr = codes + row * c.code_words, *sr = c.m > 0 ? signs + row * c.sign_words : nullptr;
      const float nu = ld_norm(db.norm, row, c.norm16), ga = c.m > 0 ? ld_norm(db.rnorm, row, c.norm16) : 0.f;
      if constexpr (POLAR)
        polar_scores<kSrQ>(c, cr, sr, nu, ga, qs, ps, ptab, sc);
      else
        estimate_scores<kSrQ>(c, cr, sr, nu, ga, qs, ps, cent, sc);
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

// ------------------------------------------------------------------ large k (32 < k <= 1024)
// A query's running top-k cannot live one entry per lane.  Each query (one warp) keeps, in shared
// memory, a buffer of kBkCap (score, index) pairs: its current top-k in [0, k), sorted best first,
// then the pending candidates that beat the current k-th entry.  When the pending part could
// overflow, and at the end, the warp sorts the occupied prefix (bitonic, rounded up to a power of
// two; every unused entry holds the sentinel (-inf, INT64_MAX)) and keeps the first k.
constexpr int kBkThreads = 128;   // rows scored per block of the scan: one per thread
constexpr int kBkQ = kBkThreads / 32;  // queries per CTA: one warp each
constexpr int kBkCap = 2048;      // per-query buffer entries (k <= 1024 leaves >= 1024 pending)

// Sort s/ix[0, n) best first by (score desc, index asc); n a power of two <= kBkCap; one warp.
__device__ __forceinline__ void warp_bitonic_best_first(float *s, int64_t *ix, int n) {
  const int lane = threadIdx.x & 31;
  for (int k2 = 2; k2 <= n; k2 <<= 1)
    for (int j = k2 >> 1; j > 0; j >>= 1) {
      for (int i = lane; i < n; i += 32) {
        const int l = i ^ j;
        if (l > i) {
          const float a = s[i], b = s[l];
          const int64_t ai = ix[i], bi = ix[l];
          // blocks with (i & k2) == 0 end best first, the others worst first
          const bool best_first = (i & k2) == 0;
          if (best_first ? tq_better(b, bi, a, ai) : tq_better(a, ai, b, bi)) {
            s[i] = b; s[l] = a;
            ix[i] = bi; ix[l] = ai;
          }
        }
      }
      __syncwarp();
    }
}

__device__ __forceinline__ int pow2_at_least(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// Running top-k of one query (one warp) in its shared-memory buffer.
struct BigTopK {
  float *s;
  int64_t *ix;
  int k, cnt;
  float ts;   // current k-th entry (sentinel until k candidates were seen)
  int64_t ti;

  __device__ void init(float *s_, int64_t *ix_, int k_) {
    s = s_; ix = ix_; k = k_; cnt = 0;
    ts = -INFINITY; ti = INT64_MAX;
    for (int i = threadIdx.x & 31; i < kBkCap; i += 32) {
      s[i] = -INFINITY;
      ix[i] = INT64_MAX;
    }
    __syncwarp();
  }
  // Keep the first k of the sorted occupied prefix; reset the rest to the sentinel.
  __device__ void compact() {
    const int n = pow2_at_least(k + cnt);
    warp_bitonic_best_first(s, ix, n);
    for (int i = k + (threadIdx.x & 31); i < n; i += 32) {
      s[i] = -INFINITY;
      ix[i] = INT64_MAX;
    }
    __syncwarp();
    ts = s[k - 1];
    ti = ix[k - 1];
    cnt = 0;
  }
  // One candidate per lane; those that beat the k-th entry join the pending part.
  __device__ void offer(float cs, int64_t ci, bool valid) {
    const int lane = threadIdx.x & 31;
    const bool take = valid && tq_better(cs, ci, ts, ti);
    const unsigned m = __ballot_sync(TQ_FULL_MASK, take);
    if (take) {
      const int pos = k + cnt + __popc(m & ((1u << lane) - 1u));
      s[pos] = cs;
      ix[pos] = ci;
    }
    cnt += __popc(m);
    __syncwarp();
    if (k + cnt + 32 > kBkCap) compact();
  }
};

template <bool POLAR>
__global__ void __launch_bounds__(kBkThreads)
search_bigk_scan_kernel(TqConsts c, const float *__restrict__ qr, const float *__restrict__ p, int nq,
                        tq_packed db, int64_t n, int k, int64_t rows_per_shard, int shards,
                        float *__restrict__ cand_s, int64_t *__restrict__ cand_i) {
  extern __shared__ __align__(16) float sm[];
  int64_t *bix = reinterpret_cast<int64_t *>(sm);   // [kBkQ][kBkCap]
  float *bsc = reinterpret_cast<float *>(bix + kBkQ * kBkCap);  // [kBkQ][kBkCap]
  float *qs = bsc + kBkQ * kBkCap;                   // [d][kBkQ]
  float *ps = qs + c.d * kBkQ;                       // [m][kBkQ]
  float *cent = ps + c.m * kBkQ;                     // [16]
  float *tile = cent + TQ_MAX_LEVELS;                // [kBkQ][kBkThreads]
  __shared__ PolarTab ptab;                          // PolarQuant contexts: the angle tables
  const int shard = blockIdx.x;
  const int q0 = blockIdx.y * kBkQ;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (POLAR) polar_tab_stage(ptab, c.polar_tab, tid, kBkThreads);
  for (int i = tid; i < c.d * kBkQ; i += kBkThreads) {
    const int j = i / kBkQ, q = i % kBkQ;
    qs[i] = (q0 + q < nq) ? qr[(int64_t)(q0 + q) * c.d + j] : 0.f;
  }
  for (int i = tid; i < c.m * kBkQ; i += kBkThreads) {
    const int j = i / kBkQ, q = i % kBkQ;
    ps[i] = (q0 + q < nq) ? p[(int64_t)(q0 + q) * c.m + j] : 0.f;
  }
  if (tid < TQ_MAX_LEVELS) cent[tid] = c.centroids[tid];
  BigTopK top;
  top.init(bsc + warp * kBkCap, bix + warp * kBkCap, k);
  __syncthreads();

  const int64_t r_begin = (int64_t)shard * rows_per_shard;
  const int64_t r_end = min(n, r_begin + rows_per_shard);
  const uint32_t *codes = static_cast<const uint32_t *>(db.codes);
  const uint32_t *signs = static_cast<const uint32_t *>(db.signs);
  const bool active = q0 + warp < nq;
  for (int64_t r0 = r_begin; r0 < r_end; r0 += kBkThreads) {
    const int64_t row = r0 + tid;
    float sc[kBkQ];
    if (row < r_end) {
      const uint32_t *cr = codes + row * c.code_words, *sr = c.m > 0 ? signs + row * c.sign_words : nullptr;
      const float nu = ld_norm(db.norm, row, c.norm16), ga = c.m > 0 ? ld_norm(db.rnorm, row, c.norm16) : 0.f;
      if constexpr (POLAR)
        polar_scores<kBkQ>(c, cr, sr, nu, ga, qs, ps, ptab, sc);
      else
        estimate_scores<kBkQ>(c, cr, sr, nu, ga, qs, ps, cent, sc);
    } else {
#pragma unroll
      for (int q = 0; q < kBkQ; ++q) sc[q] = -INFINITY;
    }
#pragma unroll
    for (int q = 0; q < kBkQ; ++q) tile[q * kBkThreads + tid] = sc[q];
    __syncthreads();
    if (active) {
#pragma unroll
      for (int ch = 0; ch < kBkThreads / 32; ++ch) {
        const int idx = ch * 32 + lane;
        const int64_t rr = r0 + idx;
        top.offer(tile[warp * kBkThreads + idx], rr, rr < r_end);
      }
    }
    __syncthreads();
  }
  if (active) {
    top.compact();
    const int64_t o = ((int64_t)(q0 + warp) * shards + shard) * k;
    for (int i = lane; i < k; i += 32) {
      cand_s[o + i] = top.s[i];
      cand_i[o + i] = top.ix[i];
    }
  }
}

// Reduce each query's shards x k candidates (each shard's list best first) to its top k.
__global__ void __launch_bounds__(kBkThreads)
search_bigk_merge_kernel(int nq, int shards, int k, const float *__restrict__ cand_s,
                         const int64_t *__restrict__ cand_i, float *__restrict__ out_s,
                         int64_t *__restrict__ out_i) {
  extern __shared__ __align__(16) float sm[];
  int64_t *bix = reinterpret_cast<int64_t *>(sm);
  float *bsc = reinterpret_cast<float *>(bix + kBkQ * kBkCap);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = blockIdx.x * kBkQ + warp;
  if (q >= nq) return;  // whole warps leave; no block-wide barrier follows
  BigTopK top;
  top.init(bsc + warp * kBkCap, bix + warp * kBkCap, k);
  for (int sh = 0; sh < shards; ++sh) {
    const int64_t base = ((int64_t)q * shards + sh) * k;
    for (int c0 = 0; c0 < k; c0 += 32) {
      const int i = c0 + lane;
      const bool in = i < k;
      const float cs = in ? cand_s[base + i] : -INFINITY;
      const int64_t ci = in ? cand_i[base + i] : INT64_MAX;
      const bool valid = in && ci != INT64_MAX;
      // a shard's list is sorted: once none of 32 beats the k-th entry, the rest cannot either
      const bool beats = valid && tq_better(cs, ci, top.ts, top.ti);
      if (!__any_sync(TQ_FULL_MASK, beats)) break;
      top.offer(cs, ci, valid);
    }
  }
  top.compact();
  for (int i = lane; i < k; i += 32) {
    out_s[(int64_t)q * k + i] = top.s[i];
    out_i[(int64_t)q * k + i] = top.ix[i];
  }
}

}  // namespace

int search_bigk_shards(int nq, int64_t n) {
  const int64_t qtiles = (nq + kBkQ - 1) / kBkQ;
  int64_t shards = qtiles > 0 ? (2 * 148 + qtiles - 1) / qtiles : 1;
  const int64_t max_shards = (n + kBkThreads - 1) / kBkThreads;
  if (shards > max_shards) shards = max_shards;
  if (shards < 1) shards = 1;
  return (int)shards;
}

cudaError_t launch_search_bigk(const TqConsts &c, int shards, const float *qr, const float *p, int nq,
                               const tq_packed &db, int64_t n, int k, float *cand_s, int64_t *cand_i,
                               float *out_s, int64_t *out_i, cudaStream_t st) {
  if (nq <= 0) return cudaSuccess;
  const size_t buf = (size_t)kBkQ * kBkCap * (sizeof(float) + sizeof(int64_t));
  const size_t smem = buf + sizeof(float) * ((size_t)(c.d + c.m) * kBkQ + TQ_MAX_LEVELS + kBkQ * kBkThreads);
  auto scan = c.polar ? search_bigk_scan_kernel<true> : search_bigk_scan_kernel<false>;
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(scan), (int)smem);
  if (e != cudaSuccess) return e;
  e = tq_smem_limit(reinterpret_cast<const void *>(search_bigk_merge_kernel), (int)buf);
  if (e != cudaSuccess) return e;
  const int64_t rows_per_shard = (n + shards - 1) / shards;
  dim3 grid((unsigned)shards, (unsigned)((nq + kBkQ - 1) / kBkQ));
  tq_prof_begin(TQK_SEARCH_SCAN, st);
  scan<<<grid, kBkThreads, smem, st>>>(c, qr, p, nq, db, n, k, rows_per_shard, shards, cand_s, cand_i);
  tq_prof_end(TQK_SEARCH_SCAN, st);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  tq_prof_begin(TQK_SEARCH_MERGE, st);
  search_bigk_merge_kernel<<<(unsigned)((nq + kBkQ - 1) / kBkQ), kBkThreads, buf, st>>>(nq, shards, k, cand_s,
                                                                                        cand_i, out_s, out_i);
  tq_prof_end(TQK_SEARCH_MERGE, st);
  return cudaGetLastError();
}

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
  auto scan = c.polar ? search_scan_kernel<true> : search_scan_kernel<false>;
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(scan), (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)plan.shards, (unsigned)((nq + kSrQ - 1) / kSrQ));
  tq_prof_begin(TQK_SEARCH_SCAN, st);
  scan<<<grid, kSrThreads, smem, st>>>(c, qr, p, nq, db, n, k, rows_per_shard, plan.shards, cand_s, cand_i);
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
