// QJL projection Z = R S^T, with two epilogues:
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


// Tensor-core variant for d % 32 == 0 and m % 64 == 0: Z = R S^T with mma.sync m16n8k8 TF32 and
// the 3-pass split x = hi + lo (hi = tf32(x), lo = tf32(x - hi)); a_hi b_hi + a_hi b_lo + a_lo b_hi
// keeps about 22 mantissa bits, the accuracy of the fp32 FMA kernel above, with fp32 accumulation.
// CTA tile 128 rows x 64 columns, 8 warps of 32 x 32, K staged 32 at a time through two
// cp.async buffers (rows padded to 36 floats: fragment loads are bank-conflict free).
constexpr int kMR = 128, kMC = 64, kMK = 32, kMS = kMK + 4;

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
  hi = to_tf32(x);
  lo = to_tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp16(float *dst, const float *src, bool ok) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(sa), "l"(src), "r"(ok ? 16 : 0) : "memory");
}

template <int EP>
__global__ void __launch_bounds__(256)
project_mma_kernel(TqConsts c, const float *__restrict__ R, int64_t n, const int64_t *__restrict__ slots,
                   int64_t capacity, uint32_t *__restrict__ signs, float *__restrict__ zout) {
  extern __shared__ __align__(16) float psm[];  // As [2][kMR * kMS], then Bs [2][kMC * kMS]
  float (*As)[kMR * kMS] = reinterpret_cast<float (*)[kMR * kMS]>(psm);
  float (*Bs)[kMC * kMS] = reinterpret_cast<float (*)[kMC * kMS]>(psm + 2 * kMR * kMS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, t = lane & 3;
  const int wr = warp >> 1, wc = warp & 1;  // warp tile: rows 32 wr.., columns 32 wc..
  const int64_t row0 = (int64_t)blockIdx.x * kMR;
  const int col0 = blockIdx.y * kMC;
  const int d = c.d, m = c.m;

  auto stage = [&](int buf, int k0) {
    // A: 128 rows x 32 k = 1024 granules, 4 per thread; B: 64 x 32 = 512 granules, 2 per thread
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int g = tid + 256 * i, r = g >> 3, kq = (g & 7) * 4;
      const int64_t gr = row0 + r;
      cp16(&As[buf][r * kMS + kq], R + (gr < n ? gr : 0) * d + k0 + kq, gr < n);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int g = tid + 256 * i, r = g >> 3, kq = (g & 7) * 4;
      cp16(&Bs[buf][r * kMS + kq], c.S + (int64_t)(col0 + r) * d + k0 + kq, true);
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  };

  float acc[2][4][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  const int nk = d / kMK;
  stage(0, 0);
  for (int kc = 0; kc < nk; ++kc) {
    const int cur = kc & 1;
    if (kc + 1 < nk) {
      stage(cur ^ 1, (kc + 1) * kMK);
      asm volatile("cp.async.wait_group 1;\n" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    }
    __syncthreads();
    const float *A = As[cur], *B = Bs[cur];
#pragma unroll
    for (int kk = 0; kk < kMK; kk += 8) {
      uint32_t ah[2][4], al[2][4], bh[4][2], bl[4][2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = 32 * wr + 16 * i + gid;
        split_tf32(A[r * kMS + kk + t], ah[i][0], al[i][0]);
        split_tf32(A[(r + 8) * kMS + kk + t], ah[i][1], al[i][1]);
        split_tf32(A[r * kMS + kk + t + 4], ah[i][2], al[i][2]);
        split_tf32(A[(r + 8) * kMS + kk + t + 4], ah[i][3], al[i][3]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = 32 * wc + 8 * j + gid;
        split_tf32(B[cc * kMS + kk + t], bh[j][0], bl[j][0]);
        split_tf32(B[cc * kMS + kk + t + 4], bh[j][1], bl[j][1]);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mma_tf32(acc[i][j], al[i], bh[j][0], bh[j][1]);
          mma_tf32(acc[i][j], ah[i], bl[j][0], bl[j][1]);
          mma_tf32(acc[i][j], ah[i], bh[j][0], bh[j][1]);
        }
    }
    __syncthreads();  // the buffer is refilled next
  }

  // acc[i][j]: rows 32 wr + 16 i + gid (e 0, 1) and + 8 (e 2, 3); columns 32 wc + 8 j + 2 t + (e & 1)
  if (EP == PROJ_DENSE) {
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t r = row0 + 32 * wr + 16 * i + gid + 8 * h;
        if (r >= n) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = col0 + 32 * wc + 8 * j + 2 * t;
          *reinterpret_cast<float2 *>(zout + r * m + col) = make_float2(acc[i][j][2 * h], acc[i][j][2 * h + 1]);
        }
      }
  } else {
    // the warp tile's 32 columns are one sign word per row: each lane sets its 8 bits, the 4
    // lanes of a row OR them together
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t w = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          w |= (acc[i][j][2 * h] >= 0.f ? 1u : 0u) << (8 * j + 2 * t);
          w |= (acc[i][j][2 * h + 1] >= 0.f ? 1u : 0u) << (8 * j + 2 * t + 1);
        }
        w |= __shfl_xor_sync(TQ_FULL_MASK, w, 1);
        w |= __shfl_xor_sync(TQ_FULL_MASK, w, 2);
        const int64_t r = row0 + 32 * wr + 16 * i + gid + 8 * h;
        if (t == 0 && r < n) {
          const int64_t slot = slots ? slots[r] : r;
          if (slot >= 0 && slot < capacity) signs[slot * c.sign_words + ((col0 + 32 * wc) >> 5)] = w;
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
  if (c.d % kMK == 0 && c.m % kMC == 0) {
    // tensor cores (3 x TF32): the projection of large batches and of the search queries
    dim3 g2((unsigned)((n + kMR - 1) / kMR), (unsigned)(c.m / kMC));
    const int smem = (int)(sizeof(float) * 2 * (kMR + kMC) * kMS);
    cudaError_t e;
    if (ep == PROJ_SIGNS) {
      e = tq_smem_limit(reinterpret_cast<const void *>(project_mma_kernel<PROJ_SIGNS>), smem);
      if (e == cudaSuccess)
        project_mma_kernel<PROJ_SIGNS><<<g2, 256, smem, st>>>(c, R, n, slots, capacity, signs, zout);
    } else {
      e = tq_smem_limit(reinterpret_cast<const void *>(project_mma_kernel<PROJ_DENSE>), smem);
      if (e == cudaSuccess)
        project_mma_kernel<PROJ_DENSE><<<g2, 256, smem, st>>>(c, R, n, slots, capacity, signs, zout);
    }
    if (e != cudaSuccess) {
      tq_prof_end(kind, st);
      return e;
    }
  } else if (ep == PROJ_SIGNS) {
    project_kernel<PROJ_SIGNS><<<grid, 256, 0, st>>>(c, R, n, slots, capacity, signs, zout);
  } else {
    project_kernel<PROJ_DENSE><<<grid, 256, 0, st>>>(c, R, n, slots, capacity, signs, zout);
  }
  tq_prof_end(kind, st);
  return cudaGetLastError();
}
