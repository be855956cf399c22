// tq_scores: estimated inner products of prepared queries with every packed key.
//   out[i][k] = nu_k ( <q'_i, c[code_k]> + sqrt(pi/2)/m gamma_k sum_j (2 bit_kj - 1) p_ij )
// ("谷歌 TurboQuant 深度拆解" 第二部分 第二步 and 第六部分 "无偏估计的数学保证").
// One thread per key and 8 queries per CTA; the prepared queries sit in shared memory as
// [coordinate][query] so that all lanes read the same coordinate (broadcast) at once.  The CTA's
// 128 packed key rows are one contiguous span per array: they are staged into shared memory with
// coalesced 16-byte loads, one padding word per row so that lanes reading their own rows hit
// distinct banks.
#include "device_common.cuh"

namespace {

constexpr int kScThreads = 128;
constexpr int kScQ = 8;

__global__ void __launch_bounds__(kScThreads)
scores_kernel(TqConsts c, const float *__restrict__ qr, const float *__restrict__ p, int nq,
              tq_packed keys, int64_t n, float *__restrict__ out) {
  extern __shared__ float sm[];
  float *qs = sm;                       // [d][kScQ]
  float *ps = qs + c.d * kScQ;          // [m][kScQ]
  float *cent = ps + c.m * kScQ;        // [16]
  const int q0 = blockIdx.y * kScQ;
  for (int i = threadIdx.x; i < c.d * kScQ; i += blockDim.x) {
    const int j = i / kScQ, q = i % kScQ;
    qs[i] = (q0 + q < nq) ? qr[(int64_t)(q0 + q) * c.d + j] : 0.f;
  }
  for (int i = threadIdx.x; i < c.m * kScQ; i += blockDim.x) {
    const int j = i / kScQ, q = i % kScQ;
    ps[i] = (q0 + q < nq) ? p[(int64_t)(q0 + q) * c.m + j] : 0.f;
  }
  if (threadIdx.x < TQ_MAX_LEVELS) cent[threadIdx.x] = c.centroids[threadIdx.x];
  const int64_t k0 = (int64_t)blockIdx.x * kScThreads;
  const int rows = n - k0 < kScThreads ? (int)(n - k0) : kScThreads;
  const int cst = c.code_words + 1, sst = c.sign_words + 1;
  uint32_t *ct = reinterpret_cast<uint32_t *>(cent + TQ_MAX_LEVELS);  // [rows][code_words + 1]
  uint32_t *stl = ct + kScThreads * cst;                              // [rows][sign_words + 1]
  {
    // rows are 16-byte multiples, so the span is a whole number of uint4
    const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint32_t *>(keys.codes) + k0 * c.code_words);
    const int q4 = c.code_words >> 2, tot = rows * q4;
    for (int i = threadIdx.x; i < tot; i += kScThreads) {
      const uint4 u = src[i];
      uint32_t *dst = ct + (i / q4) * cst + (i % q4) * 4;
      dst[0] = u.x; dst[1] = u.y; dst[2] = u.z; dst[3] = u.w;
    }
  }
  if (c.m > 0) {
    const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint32_t *>(keys.signs) + k0 * c.sign_words);
    const int q4 = c.sign_words >> 2, tot = rows * q4;
    for (int i = threadIdx.x; i < tot; i += kScThreads) {
      const uint4 u = src[i];
      uint32_t *dst = stl + (i / q4) * sst + (i % q4) * 4;
      dst[0] = u.x; dst[1] = u.y; dst[2] = u.z; dst[3] = u.w;
    }
  }
  __syncthreads();
  const int64_t key = k0 + threadIdx.x;
  if (key >= n) return;
  const uint32_t *crow = ct + threadIdx.x * cst;
  const uint32_t *srow = c.m > 0 ? stl + threadIdx.x * sst : nullptr;
  const float gamma = c.m > 0 ? ld_norm(keys.rnorm, key, c.norm16) : 0.f;
  float sc[kScQ];
  estimate_scores<kScQ>(c, crow, srow, ld_norm(keys.norm, key, c.norm16), gamma, qs, ps, cent, sc);
#pragma unroll
  for (int q = 0; q < kScQ; ++q)
    if (q0 + q < nq) out[(int64_t)(q0 + q) * n + key] = sc[q];
}

}  // namespace

cudaError_t launch_scores(const TqConsts &c, const float *qr, const float *p, int nq,
                          const tq_packed &keys, int64_t n, float *out, cudaStream_t st) {
  if (n <= 0 || nq <= 0) return cudaSuccess;
  const size_t smem = sizeof(float) * ((size_t)(c.d + c.m) * kScQ + TQ_MAX_LEVELS) +
                      sizeof(uint32_t) * (size_t)kScThreads * (c.code_words + 1 + (c.m > 0 ? c.sign_words + 1 : 0));
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(scores_kernel), (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((n + kScThreads - 1) / kScThreads), (unsigned)((nq + kScQ - 1) / kScQ));
  tq_prof_begin(TQK_SCORES, st);
  scores_kernel<<<grid, kScThreads, smem, st>>>(c, qr, p, nq, keys, n, out);
  tq_prof_end(TQK_SCORES, st);
  return cudaGetLastError();
}
