// Bulk encode at d = 128 with one row per thread ("谷歌 TurboQuant 深度拆解" 第二部分 第一步 and
// 第二步; "TurboQuant 学习路径" 二.2):
//
//   nu = ||x||, y = H (D x) (the unnormalised Walsh-Hadamard transform; y / (sqrt(d) nu) is the
//   rotated unit vector), code_j = #{i : t_i <= y_j / (sqrt(d) nu)}, r = y / (sqrt(d) nu) - c[code],
//   gamma = ||r||; with a structured QJL matrix S = P H D2: bit_i = [(H (D2 r))_i >= 0].
//
// A thread holds its whole row in registers, so the transform, the thresholds and the bit-plane
// packing need no shuffles, shared-memory atomics or residual round trip through memory.  The
// comparison is made against the thresholds scaled by sqrt(d) nu instead of scaling the row
// (t_i when nu = 0, where the row is zero).  Rows are staged into shared memory with 16-byte
// cp.async copies (double-buffered tiles of 128 rows, row stride padded so that a thread's
// 16-byte reads of its own row are free of bank conflicts), CTAs loop over tiles.
//
// Token-block value layout (TQ_LAYOUT_BLOCK16): the 32 rows of a warp are two whole 16-slot
// blocks; the words of a block are assembled with ballots across the lanes (lane = token) and
// stored whole, so this path takes only full blocks of rows written to slots equal to their row
// index; the caller encodes a ragged tail (or explicit slots) with the general kernel.
#include "device_common.cuh"
#include "tc_common.cuh"

namespace {

constexpr int kTD = 128;              // vector length served here
constexpr int kTRows = 128;           // rows per tile = threads per CTA
constexpr int kTpad = 16;             // bytes of padding per staged row

template <int DT>
struct TprRow {
  static constexpr int bytes = DT == TQ_F32 ? 4 * kTD : 2 * kTD;
  static constexpr int stride = bytes + kTpad;
  static constexpr int chunks = bytes / 16;
};

__device__ __forceinline__ void fwht128(float (&v)[kTD]) {
#pragma unroll
  for (int h = 1; h < kTD; h <<= 1)
#pragma unroll
    for (int j = 0; j < kTD; ++j)
      if ((j & h) == 0) {
        const float a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
}

// Issue the cp.async copies of tile rows [r0, r0 + kTRows) into `dst` (rows past n are skipped).
template <int DT>
__device__ __forceinline__ void tpr_stage(const char *__restrict__ x, int64_t ld_bytes, int64_t n, int64_t r0,
                                          unsigned char *dst) {
  using R = TprRow<DT>;
  for (int c = threadIdx.x; c < kTRows * R::chunks; c += kTRows) {
    const int row = c / R::chunks, col = c % R::chunks;
    if (r0 + row < n) cp_async16(dst + row * R::stride + col * 16, x + (r0 + row) * ld_bytes + col * 16);
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int DT>
__device__ __forceinline__ void tpr_load(const unsigned char *rowp, float (&v)[kTD]) {
  if constexpr (DT == TQ_F32) {
#pragma unroll
    for (int c = 0; c < kTD / 4; ++c) {
      const float4 f = *reinterpret_cast<const float4 *>(rowp + 16 * c);
      v[4 * c] = f.x; v[4 * c + 1] = f.y; v[4 * c + 2] = f.z; v[4 * c + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < kTD / 8; ++c) {
      const uint4 u = *reinterpret_cast<const uint4 *>(rowp + 16 * c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * c + 2 * e] = __uint_as_float(w[e] << 16);
        v[8 * c + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
    }
  }
}

struct TprArgs {
  const char *x;
  int64_t ld_bytes;
  int64_t n;
  const int64_t *slots;  // ROWS layout only (NULL: slot = row)
  int64_t capacity;
  uint32_t *codes;
  float *norm, *rnorm;
  uint32_t *signs;       // structured QJL only
};

// One thread per row.  BITS: MSE bits; BLK: token-block layout (full blocks, slot = row);
// SRHT: structured QJL signs of the residual.
template <int DT, int BITS, bool BLK, bool SRHT>
__global__ void __launch_bounds__(kTRows)
encode_tpr_kernel(TqConsts c, TprArgs a) {
  using R = TprRow<DT>;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float sgn[kTD], sgn2[kTD], cen[TQ_MAX_LEVELS];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int j = tid; j < kTD; j += kTRows) {
    sgn[j] = c.signs[j];
    sgn2[j] = SRHT ? c.qjl_signs[j] : 0.f;
  }
  if (tid < TQ_MAX_LEVELS) cen[tid] = c.centroids[tid];
  constexpr int L = 1 << BITS;
  float thr[L - 1];
#pragma unroll
  for (int i = 0; i < L - 1; ++i) thr[i] = c.thresholds[i];
  const float sqrtd = 1.f / c.inv_sqrt_d;
  const int64_t ntiles = (a.n + kTRows - 1) / kTRows;
  int64_t tile = blockIdx.x;
  int buf = 0;
  if (tile < ntiles) tpr_stage<DT>(a.x, a.ld_bytes, a.n, tile * kTRows, smem);
  for (; tile < ntiles; tile += gridDim.x) {
    const int64_t next = tile + gridDim.x;
    if (next < ntiles) {
      tpr_stage<DT>(a.x, a.ld_bytes, a.n, next * kTRows, smem + (buf ^ 1) * kTRows * R::stride);
      asm volatile("cp.async.wait_group 1;\n" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    }
    __syncthreads();
    const int64_t row = tile * kTRows + tid;
    const bool valid = row < a.n;
    float v[kTD];
    tpr_load<DT>(smem + buf * kTRows * R::stride + tid * R::stride, v);
    // norm, signs, transform
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kTD; ++j) ss = fmaf(v[j], v[j], ss);
    const float nu = sqrtf(ss);
#pragma unroll
    for (int j = 0; j < kTD; j += 4) {
      const float4 s4 = *reinterpret_cast<const float4 *>(sgn + j);
      v[j] *= s4.x; v[j + 1] *= s4.y; v[j + 2] *= s4.z; v[j + 3] *= s4.w;
    }
    fwht128(v);
    // codes against the scaled thresholds, bit-planes packed in registers, residual
    const float scl = nu > 0.f ? nu * sqrtd : 1.f;
    const float inv = nu > 0.f ? 1.f / scl : 0.f;
    float T[L - 1];
#pragma unroll
    for (int i = 0; i < L - 1; ++i) T[i] = thr[i] * scl;
    uint32_t w[BITS][kTD / 32];
#pragma unroll
    for (int P = 0; P < BITS; ++P)
#pragma unroll
      for (int q = 0; q < kTD / 32; ++q) w[P][q] = 0u;
    float rr = 0.f;
#pragma unroll
    for (int j = 0; j < kTD; ++j) {
      int code = 0;
#pragma unroll
      for (int i = 0; i < L - 1; ++i) code += v[j] >= T[i] ? 1 : 0;
#pragma unroll
      for (int P = 0; P < BITS; ++P) w[P][j >> 5] |= (uint32_t)((code >> P) & 1) << (j & 31);
      if constexpr (SRHT) {
        const float r = fmaf(v[j], inv, -cen[code]);  // residual, rotated domain
        v[j] = r;
        rr = fmaf(r, r, rr);
      }
    }
    if constexpr (BLK) {
      // two whole blocks per warp (slot = row); block words assembled with ballots, lane q of a
      // 32-word group keeps word q
      const int64_t wrow0 = tile * kTRows + 32 * warp;
      if (wrow0 < a.n) {  // the caller passes a multiple of 32 rows... or of 16: guard each block
        const bool twoblk = wrow0 + 16 < a.n;
        uint32_t *blkA = a.codes + (wrow0 >> 4) * (int64_t)(16 * c.code_words);
        uint32_t *blkB = blkA + 16 * c.code_words;
#pragma unroll
        for (int q2 = 0; q2 < BITS / 2; ++q2)
#pragma unroll
          for (int g = 0; g < kTD / 32; ++g) {
            uint32_t kA = 0u, kB = 0u;
#pragma unroll 4
            for (int jj = 0; jj < 32; ++jj) {
              const unsigned lo = __ballot_sync(TQ_FULL_MASK, (w[2 * q2][g] >> jj) & 1u);
              const unsigned hi = __ballot_sync(TQ_FULL_MASK, (w[2 * q2 + 1][g] >> jj) & 1u);
              if (lane == jj) {
                kA = (lo & 0xFFFFu) | (hi << 16);
                kB = (lo >> 16) | (hi & 0xFFFF0000u);
              }
            }
            blkA[q2 * kTD + 32 * g + lane] = kA;
            if (twoblk) blkB[q2 * kTD + 32 * g + lane] = kB;
          }
        if constexpr (BITS & 1) {
          // the odd last plane packs coordinates 2 j' (bits 0-15) and 2 j' + 1 (bits 16-31)
#pragma unroll
          for (int g = 0; g < kTD / 64; ++g) {
            uint32_t kA = 0u, kB = 0u;
            const uint32_t we = w[BITS - 1][2 * g], wo = w[BITS - 1][2 * g + 1];
#pragma unroll 4
            for (int jj = 0; jj < 32; ++jj) {
              // coordinates 64 g + 2 jj and 64 g + 2 jj + 1: bits 2 jj, 2 jj + 1 of word 2 g (jj < 16) or 2 g + 1
              const uint32_t wd = jj < 16 ? we : wo;
              const int sh = (2 * jj) & 31;
              const unsigned ev = __ballot_sync(TQ_FULL_MASK, (wd >> sh) & 1u);
              const unsigned od = __ballot_sync(TQ_FULL_MASK, (wd >> (sh + 1)) & 1u);
              if (lane == jj) {
                kA = (ev & 0xFFFFu) | (od << 16);
                kB = (ev >> 16) | (od & 0xFFFF0000u);
              }
            }
            blkA[(BITS / 2) * kTD + 32 * g + lane] = kA;
            if (twoblk) blkB[(BITS / 2) * kTD + 32 * g + lane] = kB;
          }
        }
      }
      if (valid) a.norm[row] = nu;
    } else {
      const int64_t slot = valid ? (a.slots ? a.slots[row] : row) : -1;
      if (valid && slot >= 0 && slot < a.capacity) {
        uint4 *dst = reinterpret_cast<uint4 *>(a.codes + slot * c.code_words);
        // b planes of 4 words = the row's b * 16 bytes (code_words = 4 b at d = 128)
#pragma unroll
        for (int P = 0; P < BITS; ++P) dst[P] = make_uint4(w[P][0], w[P][1], w[P][2], w[P][3]);
        a.norm[slot] = nu;
        if constexpr (SRHT) {
          // structured QJL: z = H (D2 r), the first m signs
          a.rnorm[slot] = sqrtf(rr);
#pragma unroll
          for (int j = 0; j < kTD; j += 4) {
            const float4 s4 = *reinterpret_cast<const float4 *>(sgn2 + j);
            v[j] *= s4.x; v[j + 1] *= s4.y; v[j + 2] *= s4.z; v[j + 3] *= s4.w;
          }
          fwht128(v);
          uint32_t sb[kTD / 32];
#pragma unroll
          for (int q = 0; q < kTD / 32; ++q) {
            uint32_t m = 0u;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) m |= (v[32 * q + jj] >= 0.f ? 1u : 0u) << jj;
            sb[q] = 32 * q < c.m ? m : 0u;
          }
          *reinterpret_cast<uint4 *>(a.signs + slot * c.sign_words) = make_uint4(sb[0], sb[1], sb[2], sb[3]);
        }
      }
    }
    __syncthreads();  // this buffer is refilled two tiles from now
    buf ^= 1;
  }
}

template <int DT, int BITS, bool BLK, bool SRHT>
cudaError_t launch_tpr_t(const TqConsts &c, const TprArgs &a, cudaStream_t st) {
  using R = TprRow<DT>;
  const size_t smem = (size_t)2 * kTRows * R::stride;
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(encode_tpr_kernel<DT, BITS, BLK, SRHT>), (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntiles = (a.n + kTRows - 1) / kTRows;
  const int64_t grid = ntiles < 3 * (int64_t)sms ? ntiles : 3 * (int64_t)sms;
  tq_prof_begin(TQK_ENCODE_ROWS, st);
  encode_tpr_kernel<DT, BITS, BLK, SRHT><<<(unsigned)grid, kTRows, smem, st>>>(c, a);
  tq_prof_end(TQK_ENCODE_ROWS, st);
  return cudaGetLastError();
}

template <int DT>
cudaError_t launch_tpr_dt(const TqConsts &c, const TprArgs &a, cudaStream_t st) {
  const bool blk = c.layout == TQ_LAYOUT_BLOCK16;
  const bool srht = c.srht != 0 && c.m > 0;
#define TQ_TPR(B)                                                                       \
  case B:                                                                               \
    if (blk) return launch_tpr_t<DT, B, true, false>(c, a, st);                         \
    return srht ? launch_tpr_t<DT, B, false, true>(c, a, st) : launch_tpr_t<DT, B, false, false>(c, a, st);
  switch (c.bits) {
    TQ_TPR(1) TQ_TPR(2) TQ_TPR(3) TQ_TPR(4)
    default: return cudaErrorInvalidValue;
  }
#undef TQ_TPR
}


// A thread's row of z (tensor memory, 128 fp32 columns from `zaddr`): sign bits of its slot.
__device__ __forceinline__ void pack_signs_from_z(uint32_t zaddr, const TqConsts &c, const TprArgs &a, int64_t slot) {
  uint32_t sb[kTD / 32];
#pragma unroll
  for (int q = 0; q < kTD / 32; ++q) {
    uint32_t z0[16], z1[16];
    tmem_ld16(zaddr + 32u * q, z0);
    tmem_ld16(zaddr + 32u * q + 16u, z1);
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
    uint32_t m = 0u;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      m |= (__uint_as_float(z0[e]) >= 0.f ? 1u : 0u) << e;
      m |= (__uint_as_float(z1[e]) >= 0.f ? 1u : 0u) << (16 + e);
    }
    sb[q] = m;
  }
  if (slot >= 0) *reinterpret_cast<uint4 *>(a.signs + slot * c.sign_words) = make_uint4(sb[0], sb[1], sb[2], sb[3]);
}

// tpr_stage by the 128 threads of one group (gt = thread index within the group).
template <int DT>
__device__ __forceinline__ void tpr_stage_g(const char *__restrict__ x, int64_t ld_bytes, int64_t n, int64_t r0,
                                            unsigned char *dst, int gt) {
  using R = TprRow<DT>;
  for (int cc = gt; cc < kTRows * R::chunks; cc += kTRows) {
    const int row = cc / R::chunks, col = cc % R::chunks;
    if (r0 + row < n) cp_async16(dst + row * R::stride + col * 16, x + (r0 + row) * ld_bytes + col * 16);
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}


// ------------------------------------------------------------------ Gaussian QJL on tcgen05
// Keys with a dense Gaussian JL matrix (m = d = 128): the same front end (one row per thread), then
// z = S r on the tensor cores as three TF32 products (r_hi S_hi + r_hi S_lo + r_lo S_hi, each
// operand split as x = tf32(x) + (x - tf32(x)); the dropped r_lo S_lo term is below 2^-22 of the
// products), which keeps z within a few fp32 ulps of the fp32 dot product.
//   A = the tile's residual rows, written by their own threads into tensor memory (lane = row,
//       one column per coordinate): r_hi for the first two products, then r_lo in the same
//       columns for the third;
//   B = S_hi, S_lo in shared memory (canonical K-major layout, staged once per CTA);
//   D = z in tensor memory, read back by the row's thread for its sign bits.
// Two groups of four compute warps (thread = row = tensor-memory lane) take alternate tiles, each
// with its own 256 tensor-memory columns (residual 128, z 128) and staging buffer; warp 8 issues
// the MMAs (one thread) and owns the allocation.  A group packs its previous tile's signs before
// encoding its next tile, so while one group waits for its products the other one computes.
constexpr int kQGroups = 2;
constexpr int kQThreads = (4 * kQGroups + 1) * 32;
constexpr int kQMmaWarp = 4 * kQGroups;
constexpr uint32_t kQLbo = 128, kQSbo = 4096;  // S: 8-row x 16-byte core matrices, K-major
constexpr int kQSBytes = kTD * kTD * 4;        // one of S_hi / S_lo

template <int DT>
struct QSmem {
  static constexpr size_t x = 0;  // one staged tile of rows per group
  static constexpr size_t shi = x + (size_t)kQGroups * kTRows * TprRow<DT>::stride;
  static constexpr size_t slo = shi + kQSBytes;
  static constexpr size_t bars = slo + kQSBytes;  // per group: rhi, rlo, hidone, zfull; then done
  static constexpr size_t total = bars + (size_t)(4 * kQGroups + 1) * 8;
  static_assert(shi % 128 == 0, "descriptor base alignment");
};

__device__ __forceinline__ bool qwait(uint64_t *bar, unsigned parity, volatile int *abort_flag) {
  for (int i = 0; i < (1 << 22); ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  return false;
}

__device__ __forceinline__ void group_sync(int g) {
  if (g == 0)
    asm volatile("bar.sync 1, 128;\n" ::: "memory");
  else
    asm volatile("bar.sync 2, 128;\n" ::: "memory");
}

template <int DT, int BITS>
__global__ void __launch_bounds__(kQThreads, 1)
encode_tcq_kernel(TqConsts c, TprArgs a) {
  using R = TprRow<DT>;
  using SM = QSmem<DT>;
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ float sgn[kTD], cen[TQ_MAX_LEVELS];
  __shared__ uint32_t tslot;
  __shared__ int abort_flag_s;
  volatile int *abort_flag = &abort_flag_s;
  uint64_t *gb = reinterpret_cast<uint64_t *>(smem + SM::bars);  // [group][rhi, rlo, hidone, zfull]
  uint64_t *done = gb + 4 * kQGroups;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int L = 1 << BITS;

  // S_hi and S_lo in the canonical K-major layout: (n, k) at (n/8) SBO + (k/4) LBO + (n%8) 16 + (k%4) 4
  for (int idx = tid; idx < kTD * kTD; idx += kQThreads) {
    const int n = idx / kTD, k = idx % kTD;
    const float sv = c.S[idx];
    const uint32_t hi = to_tf32(sv);
    const float lo = sv - __uint_as_float(hi);
    const uint32_t off = (uint32_t)(n >> 3) * kQSbo + (uint32_t)(k >> 2) * kQLbo + (uint32_t)(n & 7) * 16 + (uint32_t)(k & 3) * 4;
    *reinterpret_cast<uint32_t *>(smem + SM::shi + off) = hi;
    *reinterpret_cast<uint32_t *>(smem + SM::slo + off) = to_tf32(lo);
  }
  for (int jj = tid; jj < kTD; jj += kQThreads) sgn[jj] = c.signs[jj];
  if (tid < TQ_MAX_LEVELS) cen[tid] = c.centroids[tid];
  if (tid == 0) {
    for (int g = 0; g < kQGroups; ++g) {
      mbar_init(&gb[4 * g + 0], 4);
      mbar_init(&gb[4 * g + 1], 4);
      mbar_init(&gb[4 * g + 2], 1);
      mbar_init(&gb[4 * g + 3], 1);
    }
    mbar_init(done, 1);
    abort_flag_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kQMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(&tslot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // S visible to the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  const int64_t ntiles = (a.n + kTRows - 1) / kTRows;
  const int64_t mytiles = ntiles > blockIdx.x ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp == kQMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // D f32, A and B tf32, both K-major, N = 128, M = 128
      const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kTD >> 3) << 17) |
                             ((uint32_t)(kTRows >> 4) << 24);
      const uint32_t shi = smem_addr(smem + SM::shi), slo = smem_addr(smem + SM::slo);
      for (int64_t i = 0; i < mytiles; ++i) {
        const int g = (int)(i % kQGroups);
        const unsigned ph = (unsigned)((i / kQGroups) & 1);
        uint64_t *b = gb + 4 * g;
        const uint32_t rcol = tmem + 256u * g, zcol = rcol + 128u;
        if (!qwait(&b[0], ph, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int pass = 0; pass < 2; ++pass)  // r_hi S_hi, r_hi S_lo
#pragma unroll
          for (int ks = 0; ks < kTD / 8; ++ks)
            umma_tf32_ta(zcol, rcol + 8u * ks, umma_desc((pass ? slo : shi) + 2u * kQLbo * ks, kQLbo, kQSbo), idesc,
                         (pass == 0 && ks == 0) ? 0u : 1u);
        umma_commit(&b[2]);
        if (!qwait(&b[1], ph, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kTD / 8; ++ks)  // r_lo S_hi
          umma_tf32_ta(zcol, rcol + 8u * ks, umma_desc(shi + 2u * kQLbo * ks, kQLbo, kQSbo), idesc, 1u);
        umma_commit(&b[3]);
      }
      umma_commit(done);  // every MMA this thread issued has completed when `done` fires
      qwait(done, 0u, abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute: one row per thread
    const int g = warp >> 2, gt = tid & 127;  // group, row within the tile
    uint64_t *b = gb + 4 * g;
    unsigned char *xbuf = smem + SM::x + (size_t)g * kTRows * R::stride;
    const float sqrtd = 1.f / c.inv_sqrt_d;
    const uint32_t rbase = tmem + 256u * g + ((uint32_t)(32 * (warp & 3)) << 16), zbase = rbase + 128u;
    int64_t prev_slot = -1;
    bool ok = true;
    int64_t j = 0;  // this group's tiles so far
    int64_t i = g;  // local tile index
    if (i < mytiles) tpr_stage_g<DT>(a.x, a.ld_bytes, a.n, (blockIdx.x + i * gridDim.x) * kTRows, xbuf, gt);
    for (; i < mytiles; i += kQGroups, ++j) {
      const int64_t tile = blockIdx.x + i * gridDim.x;
      // this group's previous z: its signs first (its columns are then free for this tile)
      if (j > 0) {
        ok = qwait(&b[3], (unsigned)((j - 1) & 1), abort_flag);
        if (!__all_sync(TQ_FULL_MASK, ok)) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        tc_fence_after();
        pack_signs_from_z(zbase, c, a, prev_slot);
      }
      asm volatile("cp.async.wait_group 0;\n" ::: "memory");
      group_sync(g);
      const int64_t row = tile * kTRows + gt;
      const bool valid = row < a.n;
      const int64_t slot = valid ? (a.slots ? a.slots[row] : row) : -1;
      const bool store = valid && slot >= 0 && slot < a.capacity;
      float v[kTD];
      tpr_load<DT>(xbuf + gt * R::stride, v);
      group_sync(g);  // the buffer is free: stage this group's next tile
      if (i + kQGroups < mytiles)
        tpr_stage_g<DT>(a.x, a.ld_bytes, a.n, (blockIdx.x + (i + kQGroups) * gridDim.x) * kTRows, xbuf, gt);
      float ss = 0.f;
#pragma unroll
      for (int jj = 0; jj < kTD; ++jj) ss = fmaf(v[jj], v[jj], ss);
      const float nu = sqrtf(ss);
#pragma unroll
      for (int jj = 0; jj < kTD; jj += 4) {
        const float4 s4 = *reinterpret_cast<const float4 *>(sgn + jj);
        v[jj] *= s4.x; v[jj + 1] *= s4.y; v[jj + 2] *= s4.z; v[jj + 3] *= s4.w;
      }
      fwht128(v);
      const float scl = nu > 0.f ? nu * sqrtd : 1.f;
      const float inv = nu > 0.f ? 1.f / scl : 0.f;
      float T[L - 1];
#pragma unroll
      for (int k = 0; k < L - 1; ++k) T[k] = c.thresholds[k] * scl;
      uint32_t w[BITS][kTD / 32];
#pragma unroll
      for (int P = 0; P < BITS; ++P)
#pragma unroll
        for (int q = 0; q < kTD / 32; ++q) w[P][q] = 0u;
      float rr = 0.f;
#pragma unroll
      for (int jj = 0; jj < kTD; ++jj) {
        int code = 0;
#pragma unroll
        for (int k = 0; k < L - 1; ++k) code += v[jj] >= T[k] ? 1 : 0;
#pragma unroll
        for (int P = 0; P < BITS; ++P) w[P][jj >> 5] |= (uint32_t)((code >> P) & 1) << (jj & 31);
        const float r = fmaf(v[jj], inv, -cen[code]);
        v[jj] = r;
        rr = fmaf(r, r, rr);
      }
      if (store) {
        uint4 *dst = reinterpret_cast<uint4 *>(a.codes + slot * c.code_words);
#pragma unroll
        for (int P = 0; P < BITS; ++P) dst[P] = make_uint4(w[P][0], w[P][1], w[P][2], w[P][3]);
        a.norm[slot] = nu;
        a.rnorm[slot] = sqrtf(rr);
      }
      // r_hi -> tensor memory, then the first two products may start
#pragma unroll
      for (int cb = 0; cb < kTD / 16; ++cb) {
        uint32_t hv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          hv[e] = to_tf32(v[16 * cb + e]);
          v[16 * cb + e] -= __uint_as_float(hv[e]);  // r_lo from here on (exact in fp32)
        }
        tmem_st16(rbase + 16u * cb, hv);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&b[0]);
      // r_lo into the same columns once those products have read r_hi
      ok = qwait(&b[2], (unsigned)(j & 1), abort_flag);
      if (!__all_sync(TQ_FULL_MASK, ok)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < kTD / 16; ++cb) {
        uint32_t lv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) lv[e] = __float_as_uint(v[16 * cb + e]);
        tmem_st16(rbase + 16u * cb, lv);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(&b[1]);
      prev_slot = store ? slot : -1;
    }
    // the group's last tile's signs
    if (j > 0 && !*abort_flag) {
      ok = qwait(&b[3], (unsigned)((j - 1) & 1), abort_flag);
      if (__all_sync(TQ_FULL_MASK, ok)) {
        tc_fence_after();
        pack_signs_from_z(zbase, c, a, prev_slot);
      } else if (lane == 0) {
        *abort_flag = 1;
      }
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
  if (warp == kQMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(512) : "memory");
  }
}

template <int DT, int BITS>
cudaError_t launch_tcq_t(const TqConsts &c, const TprArgs &a, cudaStream_t st) {
  const size_t smem = QSmem<DT>::total;
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(encode_tcq_kernel<DT, BITS>), (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntiles = (a.n + kTRows - 1) / kTRows;
  const int64_t grid = ntiles < (int64_t)sms ? ntiles : (int64_t)sms;
  tq_prof_begin(TQK_ENCODE_QJL_TC, st);
  encode_tcq_kernel<DT, BITS><<<(unsigned)grid, kQThreads, smem, st>>>(c, a);
  tq_prof_end(TQK_ENCODE_QJL_TC, st);
  return cudaGetLastError();
}

template <int DT>
cudaError_t launch_tcq_dt(const TqConsts &c, const TprArgs &a, cudaStream_t st) {
  static_assert(QSmem<DT>::total <= 227 * 1024, "the tensor-core encode's shared memory");
  switch (c.bits) {
    case 1: return launch_tcq_t<DT, 1>(c, a, st);
    case 2: return launch_tcq_t<DT, 2>(c, a, st);
    case 3: return launch_tcq_t<DT, 3>(c, a, st);
    case 4: return launch_tcq_t<DT, 4>(c, a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool encode_tpr_eligible(const TqConsts &c, const int64_t *slots, tq_dtype dtype) {
  if (c.d != kTD) return false;
  // a dense S: m = d, bf16 rows (the tensor-core kernel's fp32 tiles would not fit shared memory)
  if (c.m > 0 && !c.srht && (c.m != kTD || dtype != TQ_BF16)) return false;
  if (c.layout == TQ_LAYOUT_BLOCK16 && slots != nullptr) return false;
  return true;
}

int64_t encode_tpr_rows(const TqConsts &c, int64_t n) {
  // the token-block layout takes whole blocks only; the tail goes to the general kernel
  return c.layout == TQ_LAYOUT_BLOCK16 ? n / 16 * 16 : n;
}

cudaError_t launch_encode_tpr(const TqConsts &c, const void *x, tq_dtype dtype, int64_t n, int64_t ld,
                              const int64_t *slots, int64_t capacity, uint32_t *codes, float *norm, float *rnorm,
                              uint32_t *signs, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  TprArgs a;
  a.x = static_cast<const char *>(x);
  a.ld_bytes = ld * (dtype == TQ_F32 ? 4 : 2);
  a.n = n;
  a.slots = slots;
  a.capacity = capacity;
  a.codes = codes;
  a.norm = norm;
  a.rnorm = rnorm;
  a.signs = signs;
  if (c.m > 0 && !c.srht) return launch_tcq_dt<TQ_BF16>(c, a, st);  // bf16 rows only (eligibility)
  return dtype == TQ_F32 ? launch_tpr_dt<TQ_F32>(c, a, st) : launch_tpr_dt<TQ_BF16>(c, a, st);
}
