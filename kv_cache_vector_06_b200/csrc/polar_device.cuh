// Device helpers of the PolarQuant first stage at d = 128 ("谷歌 TurboQuant 深度拆解" 第二部分 第一步:
// the rotated vector in recursive polar form, one radius and d - 1 angles, each angle quantized
// with the Lloyd-Max codebook of its level's law).  Codes: position p of the d code slots holds
// angle p, level 1 first (positions 0..63), then level 2 (64..95), ..., level 7 (126); position 127
// unused.  The angle tables (per level: thresholds, cos and sin of the centroids) come from the
// context and are staged in shared memory by the kernels that use them.
#pragma once

#include "device_common.cuh"

constexpr int kPolarD = 128, kPolarLevels = 7;

// first code slot of each level (level 1 at 0)
__host__ __device__ constexpr int polar_level_off(int l) { return kPolarD - (kPolarD >> (l - 1)); }

// [level][0: thresholds | 1: cos c | 2: sin c][16]
struct PolarTab {
  float v[kPolarLevels][3][16];
};

__device__ __forceinline__ void polar_tab_stage(PolarTab &tab, const float *__restrict__ src, int tid, int nthreads) {
  for (int i = tid; i < kPolarLevels * 3 * 16; i += nthreads) (&tab.v[0][0][0])[i] = src[i];
}

// Angle code at position p of a packed code row (bit planes of d = 128 bits, `bits` planes).
__device__ __forceinline__ int polar_code(const uint32_t *__restrict__ row, int p, int bits) {
  int c = 0;
  for (int P = 0; P < bits; ++P) c |= (int)((row[P * 4 + (p >> 5)] >> (p & 31)) & 1u) << P;
  return c;
}

// The unit direction y^ (rotated domain) from a row's angle codes, top down: (r_2i, r_2i+1) =
// r_i (cos c, sin c) at every level, level 7 first.
__device__ __forceinline__ void polar_reconstruct(const uint32_t *__restrict__ row, int bits, const PolarTab &tab,
                                                  float (&t)[kPolarD]) {
  t[0] = 1.f;
#pragma unroll
  for (int l = kPolarLevels; l >= 1; --l) {
    const int n = kPolarD >> l;
#pragma unroll
    for (int i = n - 1; i >= 0; --i) {
      const int c = polar_code(row, polar_level_off(l) + i, bits);
      const float r = t[i];
      t[2 * i] = r * tab.v[l - 1][1][c];
      t[2 * i + 1] = r * tab.v[l - 1][2][c];
    }
  }
}

// Coordinate j of y^ alone: the product along its path of cos (bit l-1 of j clear) or sin (set)
// of the level-l angle j >> l.
__device__ __forceinline__ float polar_coord(const uint32_t *__restrict__ row, int j, int bits, const PolarTab &tab) {
  float r = 1.f;
#pragma unroll
  for (int l = 1; l <= kPolarLevels; ++l) {
    const int c = polar_code(row, polar_level_off(l) + (j >> l), bits);
    r *= tab.v[l - 1][1 + ((j >> (l - 1)) & 1)][c];
  }
  return r;
}

// Estimated inner products of NQ prepared queries with one polar-coded key:
//   nu * ( <q', y^> + qjl_scale * gamma * sum_i (2 bit_i - 1) p_i )
// qs: [d][NQ], ps: [m][NQ] (shared).
template <int NQ>
__device__ __forceinline__ void polar_scores(const TqConsts &c, const uint32_t *code_row, const uint32_t *sign_row,
                                             float nu, float gamma, const float *qs, const float *ps,
                                             const PolarTab &tab, float out[NQ]) {
  float t[kPolarD];
  polar_reconstruct(code_row, c.bits, tab, t);
  float a[NQ], s2[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) a[q] = s2[q] = 0.f;
#pragma unroll
  for (int j = 0; j < kPolarD; ++j)
#pragma unroll
    for (int q = 0; q < NQ; ++q) a[q] = fmaf(qs[j * NQ + q], t[j], a[q]);
  if (c.m > 0) {
    for (int w = 0; w < c.m / 32; ++w) {
      const uint32_t sw = sign_row[w];
#pragma unroll 8
      for (int jj = 0; jj < 32; ++jj) {
        const float sg = ((sw >> jj) & 1u) ? 1.f : -1.f;
#pragma unroll
        for (int q = 0; q < NQ; ++q) s2[q] = fmaf(ps[(w * 32 + jj) * NQ + q], sg, s2[q]);
      }
    }
  }
  const float cg = c.qjl_scale * gamma;
#pragma unroll
  for (int q = 0; q < NQ; ++q) out[q] = nu * fmaf(cg, s2[q], a[q]);
}
