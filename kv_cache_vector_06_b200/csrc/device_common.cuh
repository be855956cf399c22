// Device helpers shared by the libtq kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_internal.h"

#define TQ_FULL_MASK 0xffffffffu

// Bit (t*d + j) of a packed code row read as 32-bit little-endian words: bit t of code_j.
__device__ __forceinline__ int code_bit(const uint32_t *row, int t, int j, int d) {
  const int pos = t * d + j;
  return (int)((row[pos >> 5] >> (pos & 31)) & 1u);
}

// Full code of coordinate j of `slot` in either packed layout (see tq_layout in tq.h).
__device__ __forceinline__ int slot_code(const uint32_t *codes, int64_t slot, int j, const TqConsts &c) {
  int code = 0;
  if (c.layout == TQ_LAYOUT_ROWS) {
    const uint32_t *row = codes + slot * c.code_words;
    for (int t = 0; t < c.bits; ++t) code |= code_bit(row, t, j, c.d) << t;
  } else {
    const uint32_t *blk = codes + (slot >> 4) * (int64_t)(16 * c.code_words);
    const int tok = (int)(slot & 15);
    for (int q = 0; q < c.bits / 2; ++q) {
      const uint32_t w = blk[q * c.d + j];
      code |= (int)((w >> tok) & 1u) << (2 * q);
      code |= (int)((w >> (16 + tok)) & 1u) << (2 * q + 1);
    }
    if (c.bits & 1) {
      const uint32_t w = blk[(c.bits / 2) * c.d + (j >> 1)];
      code |= (int)((w >> (16 * (j & 1) + tok)) & 1u) << (c.bits - 1);
    }
  }
  return code;
}

// 32 consecutive coordinates [32w, 32w+32) of bit-plane t as one word (d >= 32), or the whole
// d-bit plane t in the low d bits (d < 32; then w must be 0).
__device__ __forceinline__ uint32_t plane_word(const uint32_t *row, int t, int w, int d) {
  if (d >= 32) return row[t * (d >> 5) + w];
  const uint64_t v = (uint64_t)row[0] | ((uint64_t)row[1] << 32);
  return (uint32_t)((v >> (t * d)) & ((1ull << d) - 1ull));
}

// A stored norm (||x|| or ||r||) of slot i: fp16 or fp32 per the context.
__device__ __forceinline__ float ld_norm(const void *p, int64_t i, int half) {
  return half ? __half2float(static_cast<const __half *>(p)[i]) : static_cast<const float *>(p)[i];
}
__device__ __forceinline__ void st_norm(void *p, int64_t i, float v, int half) {
  if (half)
    static_cast<__half *>(p)[i] = __float2half_rn(fminf(v, 65504.f));
  else
    static_cast<float *>(p)[i] = v;
}

// Estimated inner products of NQ prepared queries with one packed key:
//   nu * ( sum_j q'_j c[code_j] + qjl_scale * gamma * sum_i (2 bit_i - 1) p_i )
// qs: [d][NQ] (shared), ps: [m][NQ] (shared), cent: [levels] (shared).
template <int NQ>
__device__ __forceinline__ void estimate_scores(const TqConsts &c, const uint32_t *code_row,
                                                const uint32_t *sign_row, float nu, float gamma,
                                                const float *qs, const float *ps,
                                                const float *cent, float out[NQ]) {
  float a[NQ], s2[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    a[q] = 0.f;
    s2[q] = 0.f;
  }
  const int d = c.d;
  const int nw = d >= 32 ? (d >> 5) : 1;
  const int nb = d >= 32 ? 32 : d;
  for (int w = 0; w < nw; ++w) {
    uint32_t pw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (t < c.bits) pw[t] = plane_word(code_row, t, w, d);
    for (int jj = 0; jj < nb; ++jj) {
      int code = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t) code |= (int)((pw[t] >> jj) & 1u) << t;
      const float cv = cent[code];
      const float *qj = qs + (size_t)(w * 32 + jj) * NQ;
#pragma unroll
      for (int q = 0; q < NQ; ++q) a[q] = fmaf(qj[q], cv, a[q]);
    }
  }
  if (c.m > 0) {
    const int mw = c.m >> 5;
    for (int w = 0; w < mw; ++w) {
      const uint32_t sw = sign_row[w];
#pragma unroll 8
      for (int jj = 0; jj < 32; ++jj) {
        const float sg = ((sw >> jj) & 1u) ? 1.f : -1.f;
        const float *pj = ps + (size_t)(w * 32 + jj) * NQ;
#pragma unroll
        for (int q = 0; q < NQ; ++q) s2[q] = fmaf(pj[q], sg, s2[q]);
      }
    }
  }
  const float cg = c.qjl_scale * gamma;
#pragma unroll
  for (int q = 0; q < NQ; ++q) out[q] = nu * fmaf(cg, s2[q], a[q]);
}

// (score desc, index asc) ordering used by top-k.
__device__ __forceinline__ bool tq_better(float s1, int64_t i1, float s2, int64_t i2) {
  return s1 > s2 || (s1 == s2 && i1 < i2);
}

// Warp-cooperative sorted top-k list (k <= 32): lane i < k holds the i-th best (score, index).
// Insert the candidates held one per lane (valid flags); keeps the list sorted.
__device__ __forceinline__ void warp_topk_insert(float &bs, int64_t &bi, int k, float cs,
                                                 int64_t ci, bool valid) {
  const int lane = threadIdx.x & 31;
  float ts = __shfl_sync(TQ_FULL_MASK, bs, k - 1);
  int64_t ti = __shfl_sync(TQ_FULL_MASK, bi, k - 1);
  unsigned mask = __ballot_sync(TQ_FULL_MASK, valid && tq_better(cs, ci, ts, ti));
  while (mask) {
    const int src = __ffs(mask) - 1;
    mask &= mask - 1;
    const float s = __shfl_sync(TQ_FULL_MASK, cs, src);
    const int64_t i = __shfl_sync(TQ_FULL_MASK, ci, src);
    if (!tq_better(s, i, ts, ti)) continue;  // uniform: every lane holds the same ts/ti
    const bool mine_better = lane < k && tq_better(bs, bi, s, i);
    const int pos = __popc(__ballot_sync(TQ_FULL_MASK, mine_better));
    const float us = __shfl_up_sync(TQ_FULL_MASK, bs, 1);
    const int64_t ui = __shfl_up_sync(TQ_FULL_MASK, bi, 1);
    if (lane > pos && lane < k) {
      bs = us;
      bi = ui;
    }
    if (lane == pos) {
      bs = s;
      bi = i;
    }
    ts = __shfl_sync(TQ_FULL_MASK, bs, k - 1);
    ti = __shfl_sync(TQ_FULL_MASK, bi, k - 1);
  }
}

// Copy a rows x cols fp32 row-major matrix (cols a multiple of 4) into shared memory with a row
// stride of cols + 4 floats, so that 16-byte loads of one column chunk by 8 lanes on 8
// consecutive rows fall in distinct banks.  Every thread of the block must call it.
__device__ __forceinline__ void stage_rows_padded(float *dst, const float *__restrict__ src, int rows, int cols) {
  const int c4 = cols >> 2;
  const int total = rows * c4;
  // eight independent 16-byte loads in flight per thread before any store
  for (int base = threadIdx.x; base < total; base += 8 * blockDim.x) {
    float4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int idx = base + k * blockDim.x;
      if (idx < total) {
        const int r = idx / c4, c = idx - r * c4;
        v[k] = *reinterpret_cast<const float4 *>(src + (size_t)r * cols + 4 * c);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int idx = base + k * blockDim.x;
      if (idx < total) {
        const int r = idx / c4, c = idx - r * c4;
        *reinterpret_cast<float4 *>(dst + (size_t)r * (cols + 4) + 4 * c) = v[k];
      }
    }
  }
}

// The same copy issued as asynchronous 16-byte copies (cp.async, no registers held), so that the
// caller can overlap it with other work; complete it with stage_async_wait() and a block barrier.
__device__ __forceinline__ void stage_rows_padded_async(float *dst, const float *__restrict__ src, int rows, int cols) {
  const int c4 = cols >> 2;
  const int total = rows * c4;
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
    const int r = idx / c4, c = idx - r * c4;
    const unsigned sa = (unsigned)__cvta_generic_to_shared(dst + (size_t)r * (cols + 4) + 4 * c);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(src + (size_t)r * cols + 4 * c) : "memory");
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
__device__ __forceinline__ void stage_async_wait() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Device-side status word of the library (bits of tq_device_status), one per translation unit:
// set by a kernel that gave up waiting, read and cleared from the host by tq_device_status.
static __device__ int g_tq_device_flags;
constexpr int kFlagStagingTimeout = 1;

// Host accessor for this translation unit's status word (read, optionally clear); each unit whose
// kernels set flags defines one and tq_device_status ORs them.
#define TQ_DEVICE_FLAGS_ACCESSOR(name)                                   \
  cudaError_t name(int *v, bool clear) {                                 \
    cudaError_t e = cudaMemcpyFromSymbol(v, g_tq_device_flags, sizeof(int)); \
    if (e == cudaSuccess && clear) {                                     \
      const int z = 0;                                                   \
      e = cudaMemcpyToSymbol(g_tq_device_flags, &z, sizeof(int));       \
    }                                                                    \
    return e;                                                            \
  }

// Bulk asynchronous copies (global -> this CTA's shared memory) completing on an mbarrier, and
// the bounded wait for them.  Addresses 16-byte aligned, sizes multiples of 16 bytes.
__device__ __forceinline__ unsigned smem_addr(const void *p) { return (unsigned)__cvta_generic_to_shared(p); }
// 16-byte asynchronous global -> shared copy through L2 (both addresses 16-byte aligned).
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr(smem_dst)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_arrive(uint64_t *bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, unsigned bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}
// One plain arrival (no transaction bytes).
__device__ __forceinline__ void mbar_arrive1(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for phase `parity` of `bar` to complete, giving up after about a second (each try_wait
// suspends for a bounded, hardware-defined time).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, unsigned parity) {
  for (int i = 0; i < (1 << 22); ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// 2^e as a float for e in [-126, 127].
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
  return __uint_as_float(((uint32_t)h) << 16);
}
