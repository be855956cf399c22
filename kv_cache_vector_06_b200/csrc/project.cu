// QJL projection Z = R S^T on CUDA cores (fp32 FMA), with two epilogues:
//   PROJ_SIGNS  bit_i = [z_i >= 0] packed LSB-first into 32-bit words at the row's slot
//               ("谷歌 TurboQuant 深度拆解" 第二部分 第二步: keep only the sign of each projected
//               residual coordinate; "TurboQuant 学习路径" 二.2: R_ij ~ N(0,1));
//   PROJ_DENSE  Z written as fp32 (the projected queries p = S q').
//
// Tiling: a CTA computes a 64-row x 64-column tile with 256 threads; thread (tx, ty) owns rows
// ty + 16a and columns tx + 16b (a, b < 4).  Both operands are K-contiguous (R rows are vectors,
// S rows are projection directions) and are staged through shared memory transposed to
// [k][row] in 16-wide K steps.  With this ownership, a warp's lanes 0-15 (resp. 16-31) hold 16
// consecutive columns of one row, so each sign word is two 16-bit halves of warp ballots.
#include "device_common.cuh"

namespace {

constexpr int kPT = 64;   // tile rows / cols
constexpr int kPK = 16;   // K step

template <int EP>
__global__ void __launch_bounds__(256)
project_kernel(TqConsts c, const float *__restrict__ R, int64_t n, const int64_t *__restrict__ slots,
               int64_t capacity, uint32_t *__restrict__ signs, float *__restrict__ zout) {
  __shared__ float As[kPK][kPT + 4];
  __shared__ float Bs[kPK][kPT + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t row0 = (int64_t)blockIdx.x * kPT;
  const int col0 = blockIdx.y * kPT;
  const int d = c.d, m = c.m;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

  const int lr = tid >> 2, lk = (tid & 3) * 4;  // loader: row within tile, k offset
  for (int k0 = 0; k0 < d; k0 += kPK) {
    {
      const int64_t gr = row0 + lr;
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
      if (gr < n && k0 + lk < d) t = *reinterpret_cast<const float4 *>(R + gr * d + k0 + lk);
      As[lk + 0][lr] = t.x; As[lk + 1][lr] = t.y; As[lk + 2][lr] = t.z; As[lk + 3][lr] = t.w;
    }
    {
      const int gc = col0 + lr;
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
      if (gc < m && k0 + lk < d) t = *reinterpret_cast<const float4 *>(c.S + (int64_t)gc * d + k0 + lk);
      Bs[lk + 0][lr] = t.x; Bs[lk + 1][lr] = t.y; Bs[lk + 2][lr] = t.z; Bs[lk + 3][lr] = t.w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kPK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) av[a] = As[kk][ty + 16 * a];
#pragma unroll
      for (int b = 0; b < 4; ++b) bv[b] = Bs[kk][tx + 16 * b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
    }
    __syncthreads();
  }

  if (EP == PROJ_DENSE) {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int64_t r = row0 + ty + 16 * a;
      if (r >= n) continue;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int col = col0 + tx + 16 * b;
        if (col < m) zout[r * m + col] = acc[a][b];
      }
    }
  } else {
    const int lane = tid & 31;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      unsigned bal[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int col = col0 + tx + 16 * b;
        bal[b] = __ballot_sync(TQ_FULL_MASK, col < m && acc[a][b] >= 0.f);
      }
      if (lane == 0 || lane == 16) {
        const int64_t r = row0 + ty + 16 * a;
        const int sh = lane;  // 0: low halves (row ty), 16: high halves (row ty + 1)
        if (r < n) {
          const int64_t slot = slots ? slots[r] : r;
          if (slot >= 0 && slot < capacity) {
#pragma unroll
            for (int cw = 0; cw < 2; ++cw) {
              const int colw = col0 + 32 * cw;
              if (colw >= m) continue;
              const uint32_t lo = (bal[2 * cw] >> sh) & 0xffffu;
              const uint32_t hi = (bal[2 * cw + 1] >> sh) & 0xffffu;
              signs[slot * c.sign_words + (colw >> 5)] = lo | (hi << 16);
            }
          }
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_project(const TqConsts &c, ProjEpilogue ep, const float *R, int64_t n,
                           const int64_t *slots, int64_t capacity, uint32_t *signs, float *zout,
                           cudaStream_t st) {
  if (n <= 0 || c.m <= 0) return cudaSuccess;
  dim3 grid((unsigned)((n + kPT - 1) / kPT), (unsigned)((c.m + kPT - 1) / kPT));
  const int kind = ep == PROJ_SIGNS ? TQK_QJL_PROJECT : TQK_QUERY_PROJECT;
  tq_prof_begin(kind, st);
  if (ep == PROJ_SIGNS)
    project_kernel<PROJ_SIGNS><<<grid, 256, 0, st>>>(c, R, n, slots, capacity, signs, zout);
  else
    project_kernel<PROJ_DENSE><<<grid, 256, 0, st>>>(c, R, n, slots, capacity, signs, zout);
  tq_prof_end(kind, st);
  return cudaGetLastError();
}
