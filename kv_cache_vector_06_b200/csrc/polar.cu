// PolarQuant first stage at d = 128 ("谷歌 TurboQuant 深度拆解" 第二部分 第一步 "PolarQuant——换一个坐标系来
// 看数据"; vocus.cc 第一階段): after the random rotation the vector is written in recursive polar
// form, pairs of coordinates -> (radius, angle), pairs of radii -> (radius, angle), ... down to one
// radius (the stored norm) and d - 1 angles, and every angle is quantized with the Lloyd-Max
// codebook of its level's known law (no per-block constants).
//
//   level 1:  r_i = |(y_2i, y_2i+1)|, a_i = atan2(y_2i+1, y_2i) in (-pi, pi]
//   level l:  r_i = |(r_2i, r_2i+1)| of level l - 1, a_i = atan2(r_2i+1, r_2i) in [0, pi/2]
//   codes: position p of the d code slots holds angle p, level 1 first (positions 0..63), then
//   level 2 (64..95), ..., level 7 (126); position 127 is unused (0).  Bit-plane layout as for the
//   coordinate codes.
//   reconstruction of the unit direction, top down: (r_2i, r_2i+1) = r_i (cos c, sin c), with c
//   the centroid of the angle's code; y^_2i, y^_2i+1 likewise at level 1.
//   QJL stage on r = y / ||x|| - y^ exactly as with the coordinate quantizer.
//
// One row per thread (registers); the angle tables (thresholds, cos and sin of the centroids per
// level) sit in shared memory.  The residual rows go to a workspace for the projection kernel.
#include "polar_device.cuh"

namespace {

constexpr int kPD = kPolarD, kPLevels = kPolarLevels, kPRows = 128;

__device__ __forceinline__ void fwht128p(float (&v)[kPD]) {
#pragma unroll
  for (int h = 1; h < kPD; h <<= 1)
#pragma unroll
    for (int j = 0; j < kPD; ++j)
      if ((j & h) == 0) {
        const float a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
}


template <int BITS>
__device__ __forceinline__ int angle_code(float a, const float *thr) {
  int c = 0;
#pragma unroll
  for (int i = 0; i < (1 << BITS) - 1; ++i) c += a >= thr[i] ? 1 : 0;
  return c;
}

template <int BITS>
__device__ __forceinline__ int code_at(const uint32_t (&w)[4][4], int p) {
  int c = 0;
#pragma unroll
  for (int P = 0; P < BITS; ++P) c |= (int)((w[P][p >> 5] >> (p & 31)) & 1u) << P;
  return c;
}

// y^ (unit direction, rotated domain) from the angle codes, top down
template <int BITS>
__device__ __forceinline__ void reconstruct(const uint32_t (&w)[4][4], const PolarTab &tab, float (&t)[kPD]) {
  t[0] = 1.f;
#pragma unroll
  for (int l = kPLevels; l >= 1; --l) {
    const int n = kPD >> l;  // angles of level l
#pragma unroll
    for (int i = n - 1; i >= 0; --i) {
      const int c = code_at<BITS>(w, polar_level_off(l) + i);
      const float r = t[i];
      t[2 * i] = r * tab.v[l - 1][1][c];
      t[2 * i + 1] = r * tab.v[l - 1][2][c];
    }
  }
}

template <int DT, int BITS>
__global__ void __launch_bounds__(kPRows)
encode_polar_kernel(TqConsts c, const char *__restrict__ x, int64_t ld_bytes, int64_t n, const int64_t *__restrict__ slots,
                    int64_t capacity, uint32_t *__restrict__ codes, void *__restrict__ norm, void *__restrict__ rnorm,
                    float *__restrict__ resid) {
  __shared__ PolarTab tab;
  __shared__ float sgn[kPD];
  for (int i = threadIdx.x; i < kPLevels * 3 * 16; i += kPRows) (&tab.v[0][0][0])[i] = c.polar_tab[i];
  for (int j = threadIdx.x; j < kPD; j += kPRows) sgn[j] = c.signs[j];
  __syncthreads();
  const int64_t row = (int64_t)blockIdx.x * kPRows + threadIdx.x;
  if (row >= n) return;
  const int64_t slot = slots ? slots[row] : row;
  const bool store = slot >= 0 && slot < capacity;
  auto load = [&](float (&v)[kPD]) {
    const char *rp = x + row * ld_bytes;
    if (DT == TQ_F32) {
#pragma unroll
      for (int q = 0; q < kPD / 4; ++q) {
        const float4 f = reinterpret_cast<const float4 *>(rp)[q];
        v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < kPD / 8; ++q) {
        const uint4 u = reinterpret_cast<const uint4 *>(rp)[q];
        const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[8 * q + 2 * e] = __uint_as_float(ww[e] << 16);
          v[8 * q + 2 * e + 1] = __uint_as_float(ww[e] & 0xffff0000u);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kPD; ++j) v[j] *= sgn[j];
    fwht128p(v);  // H D x: sqrt(d) times the rotated vector
  };
  float v[kPD];
  load(v);
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < kPD; ++j) ss = fmaf(v[j], v[j], ss);
  const float nu = sqrtf(ss) * c.inv_sqrt_d;  // ||x||
  // forward recursion in place: level l reads radii 2i, 2i+1 and writes radius i
  uint32_t w[4][4];
#pragma unroll
  for (int P = 0; P < 4; ++P)
#pragma unroll
    for (int q = 0; q < 4; ++q) w[P][q] = 0u;
#pragma unroll
  for (int l = 1; l <= kPLevels; ++l) {
    const int nl = kPD >> l;
#pragma unroll
    for (int i = 0; i < nl; ++i) {
      const float a0 = v[2 * i], a1 = v[2 * i + 1];
      const int code = angle_code<BITS>(atan2f(a1, a0), tab.v[l - 1][0]);
      const int p = polar_level_off(l) + i;
#pragma unroll
      for (int P = 0; P < BITS; ++P) w[P][p >> 5] |= (uint32_t)((code >> P) & 1) << (p & 31);
      v[i] = sqrtf(fmaf(a0, a0, a1 * a1));
    }
  }
  if (store) {
    uint4 *dst = reinterpret_cast<uint4 *>(codes + slot * c.code_words);
#pragma unroll
    for (int P = 0; P < BITS; ++P) dst[P] = make_uint4(w[P][0], w[P][1], w[P][2], w[P][3]);
    st_norm(norm, slot, nu, c.norm16);
  }
  if (resid == nullptr) return;
  // residual r = y / ||x|| - y^ (rotated domain): y^ first, then the row is transformed again
  reconstruct<BITS>(w, tab, v);
  float *rr_row = resid + row * kPD;
#pragma unroll
  for (int q = 0; q < kPD / 4; ++q)
    reinterpret_cast<float4 *>(rr_row)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  load(v);
  const float inv = nu > 0.f ? c.inv_sqrt_d / nu : 0.f;
  float rr = 0.f;
#pragma unroll
  for (int q = 0; q < kPD / 4; ++q) {
    const float4 yh = reinterpret_cast<const float4 *>(rr_row)[q];
    const float r0 = fmaf(v[4 * q], inv, -yh.x), r1 = fmaf(v[4 * q + 1], inv, -yh.y);
    const float r2 = fmaf(v[4 * q + 2], inv, -yh.z), r3 = fmaf(v[4 * q + 3], inv, -yh.w);
    rr = fmaf(r0, r0, fmaf(r1, r1, fmaf(r2, r2, fmaf(r3, r3, rr))));
    reinterpret_cast<float4 *>(rr_row)[q] = make_float4(r0, r1, r2, r3);
  }
  if (store) st_norm(rnorm, slot, sqrtf(rr), c.norm16);
}

// Estimated inner products with PolarQuant keys: nu ( <q', y^> + sqrt(pi/2)/m gamma <p, 2 b - 1> ).
// One thread per key, 8 prepared queries per CTA in shared memory ([coordinate][query]).
constexpr int kPQ = 8;

template <int BITS>
__global__ void __launch_bounds__(kPRows)
scores_polar_kernel(TqConsts c, const float *__restrict__ qr, const float *__restrict__ p, int nq, tq_packed keys,
                    int64_t n, float *__restrict__ out) {
  __shared__ PolarTab tab;
  __shared__ float qs[kPD * kPQ];
  extern __shared__ float ps[];  // [m][kPQ]
  const int q0 = blockIdx.y * kPQ;
  for (int i = threadIdx.x; i < kPLevels * 3 * 16; i += kPRows) (&tab.v[0][0][0])[i] = c.polar_tab[i];
  for (int i = threadIdx.x; i < kPD * kPQ; i += kPRows) {
    const int j = i / kPQ, q = i % kPQ;
    qs[i] = q0 + q < nq ? qr[(int64_t)(q0 + q) * kPD + j] : 0.f;
  }
  for (int i = threadIdx.x; i < c.m * kPQ; i += kPRows) {
    const int j = i / kPQ, q = i % kPQ;
    ps[i] = q0 + q < nq ? p[(int64_t)(q0 + q) * c.m + j] : 0.f;
  }
  __syncthreads();
  const int64_t key = (int64_t)blockIdx.x * kPRows + threadIdx.x;
  if (key >= n) return;
  const uint32_t *crow = static_cast<const uint32_t *>(keys.codes) + key * c.code_words;
  uint32_t w[4][4];
#pragma unroll
  for (int P = 0; P < 4; ++P)
#pragma unroll
    for (int q = 0; q < 4; ++q) w[P][q] = P < BITS ? crow[P * 4 + q] : 0u;
  float t[kPD];
  reconstruct<BITS>(w, tab, t);
  float acc[kPQ], s2[kPQ];
#pragma unroll
  for (int q = 0; q < kPQ; ++q) acc[q] = s2[q] = 0.f;
#pragma unroll
  for (int j = 0; j < kPD; ++j)
#pragma unroll
    for (int q = 0; q < kPQ; ++q) acc[q] = fmaf(qs[j * kPQ + q], t[j], acc[q]);
  float gamma = 0.f;
  if (c.m > 0) {
    gamma = ld_norm(keys.rnorm, key, c.norm16);
    const uint32_t *srow = static_cast<const uint32_t *>(keys.signs) + key * c.sign_words;
    for (int wd = 0; wd < c.m / 32; ++wd) {
      const uint32_t sw = srow[wd];
#pragma unroll 8
      for (int jj = 0; jj < 32; ++jj) {
        const float sg = ((sw >> jj) & 1u) ? 1.f : -1.f;
#pragma unroll
        for (int q = 0; q < kPQ; ++q) s2[q] = fmaf(ps[(wd * 32 + jj) * kPQ + q], sg, s2[q]);
      }
    }
  }
  const float nu = ld_norm(keys.norm, key, c.norm16), cg = c.qjl_scale * gamma;
#pragma unroll
  for (int q = 0; q < kPQ; ++q)
    if (q0 + q < nq) out[(int64_t)(q0 + q) * n + key] = nu * fmaf(cg, s2[q], acc[q]);
}

}  // namespace

bool polar_supported(const TqConsts &c) { return c.d == kPD && c.layout == TQ_LAYOUT_ROWS && c.bits >= 1 && c.bits <= 4; }

cudaError_t launch_encode_polar(const TqConsts &c, const void *x, tq_dtype dtype, int64_t n, int64_t ld,
                                const int64_t *slots, int64_t capacity, uint32_t *codes, void *norm, void *rnorm,
                                float *resid, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((n + kPRows - 1) / kPRows);
  const char *xp = static_cast<const char *>(x);
  const int64_t ldb = ld * (dtype == TQ_F32 ? 4 : 2);
  tq_prof_begin(TQK_ROTATE_ENCODE, st);
#define TQ_PE(B)                                                                                              \
  case B:                                                                                                     \
    if (dtype == TQ_F32)                                                                                      \
      encode_polar_kernel<TQ_F32, B><<<grid, kPRows, 0, st>>>(c, xp, ldb, n, slots, capacity, codes, norm, rnorm, resid); \
    else                                                                                                      \
      encode_polar_kernel<TQ_BF16, B><<<grid, kPRows, 0, st>>>(c, xp, ldb, n, slots, capacity, codes, norm, rnorm, resid); \
    break;
  switch (c.bits) {
    TQ_PE(1) TQ_PE(2) TQ_PE(3) TQ_PE(4)
    default: return cudaErrorInvalidValue;
  }
#undef TQ_PE
  tq_prof_end(TQK_ROTATE_ENCODE, st);
  return cudaGetLastError();
}

cudaError_t launch_scores_polar(const TqConsts &c, const float *qr, const float *p, int nq, const tq_packed &keys,
                                int64_t n, float *out, cudaStream_t st) {
  if (n <= 0 || nq <= 0) return cudaSuccess;
  dim3 grid((unsigned)((n + kPRows - 1) / kPRows), (unsigned)((nq + kPQ - 1) / kPQ));
  const size_t smem = sizeof(float) * (size_t)c.m * kPQ;
  tq_prof_begin(TQK_SCORES, st);
  switch (c.bits) {
    case 1: scores_polar_kernel<1><<<grid, kPRows, smem, st>>>(c, qr, p, nq, keys, n, out); break;
    case 2: scores_polar_kernel<2><<<grid, kPRows, smem, st>>>(c, qr, p, nq, keys, n, out); break;
    case 3: scores_polar_kernel<3><<<grid, kPRows, smem, st>>>(c, qr, p, nq, keys, n, out); break;
    case 4: scores_polar_kernel<4><<<grid, kPRows, smem, st>>>(c, qr, p, nq, keys, n, out); break;
    default: return cudaErrorInvalidValue;
  }
  tq_prof_end(TQK_SCORES, st);
  return cudaGetLastError();
}
