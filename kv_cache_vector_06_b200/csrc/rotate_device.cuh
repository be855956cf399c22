// Device body of the encode / query-rotation kernels (shared by rotate.cu and the fused decode
// step in attend_mma.cu).
#pragma once

#include "device_common.cuh"

//   nu = ||x||, u = x / nu, y = (1/sqrt d) H (D u)            ("TurboQuant 学习路径" 二.2: y = H D x;
//                                                              juejin 第二部分 第一步: random rotation)
//   code_j = #{i : t_i <= y_j}, r = y - c[code], gamma = ||r|| (juejin 第二部分 第一步 / 第二步)
//
// Lane layout: a vector is held by LPV = min(32, d/4) lanes; lane l owns the coordinates
// j = 4 (l + LPV k) + e, e in [0,4), k in [0, d / (4 LPV)), so every load and store is a 16-byte
// (fp32) or 8-byte (bf16) vector access and a warp reads whole rows coalesced.  The Walsh-
// Hadamard butterflies run inside a lane for distances 1, 2 and >= 4 LPV, and across lanes with
// __shfl_xor_sync for distances 4 .. 2 LPV (each stage of the transform is independent of the
// order in which stages are applied).  Codes are packed into bit-planes with shared-memory
// atomicOr on 4-bit groups, then written out as 16-byte words.

constexpr int kRotThreads = 256;

template <int D>
struct RotLayout {
  static constexpr int LPV = (D / 4) < 32 ? (D / 4) : 32;  // lanes per vector
  static constexpr int VPW = 32 / LPV;                     // vectors per warp
  static constexpr int KCH = D / (4 * LPV);                // 4-coordinate chunks per lane
  static constexpr int CW = ((4 * D / 8 + 15) / 16 * 16) / 4;  // max code words per row (b = 4)
};

template <int LPV>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int s = LPV / 2; s >= 1; s >>= 1) x += __shfl_xor_sync(TQ_FULL_MASK, x, s);
  return x;
}

// Unnormalised Walsh-Hadamard transform v <- H v of one vector held in the lane layout above
// (lane l of the group owns coordinates 4 (l + LPV k) + e): distances 1 and 2 inside a lane's
// 4-chunk, 4 .. 2 LPV across lanes, >= 4 LPV across the lane's chunks.
template <int D>
__device__ __forceinline__ void fwht_lanes(float (&v)[RotLayout<D>::KCH][4], int l) {
  constexpr int LPV = RotLayout<D>::LPV, KCH = RotLayout<D>::KCH;
#pragma unroll
  for (int k = 0; k < KCH; ++k) {
    const float a = v[k][0] + v[k][1], b = v[k][0] - v[k][1];
    const float p = v[k][2] + v[k][3], q = v[k][2] - v[k][3];
    v[k][0] = a + p; v[k][1] = b + q; v[k][2] = a - p; v[k][3] = b - q;
  }
#pragma unroll
  for (int s = 1; s < LPV; s <<= 1) {
    const bool hi = (l & s) != 0;
#pragma unroll
    for (int k = 0; k < KCH; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float o = __shfl_xor_sync(TQ_FULL_MASK, v[k][e], s);
        v[k][e] = hi ? (o - v[k][e]) : (v[k][e] + o);
      }
  }
#pragma unroll
  for (int h = 1; h < KCH; h <<= 1)
#pragma unroll
    for (int k = 0; k < KCH; ++k)
      if ((k & h) == 0)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = v[k][e], b = v[k + h][e];
          v[k][e] = a + b;
          v[k + h][e] = a - b;
        }
}

// The encode / query-rotation work of one block of kRotThreads threads: rows of block `vblock`.
// `sS` is dynamic shared memory of at least 128 x 132 floats when d = m = 128 and `fsigns` is set
// (the fused projection stages S there), or null to read S rows from global memory (same
// arithmetic, same results); every thread of the block must call it with the same
// arguments.  With `one_vec` (d = m = 128, fused projection) the block encodes the single row
// `vblock`: warp 0 rotates and quantizes it and warps 0-3 share its projection, 32 rows each (the
// same arithmetic as one warp doing all 128).
template <int D>
__device__ __forceinline__ void rotate_rows(const TqConsts &c, int mode, const void *__restrict__ x, int dtype,
                                            int64_t n, int64_t ld, const int64_t *__restrict__ slots,
                                            int64_t capacity, uint32_t *__restrict__ codes,
                                            void *__restrict__ norm, void *__restrict__ rnorm,
                                            float *__restrict__ resid, uint32_t *__restrict__ fsigns,
                                            int64_t vblock, float *sS, bool one_vec = false) {
  using Lay = RotLayout<D>;
  constexpr int LPV = Lay::LPV, VPW = Lay::VPW, KCH = Lay::KCH;
  __shared__ uint32_t stage[kRotThreads / 32][VPW][Lay::CW];
  __shared__ float rbuf[kRotThreads / 32][D >= 128 ? D : 1];  // residual, fused projection

  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  // fused projection with S staged in shared memory (d = m = 128; row stride 132 floats)
  const bool staged = D == 128 && fsigns != nullptr && c.m == 128 && !c.srht && sS != nullptr;
  if (staged) stage_rows_padded_async(sS, c.S, 128, 128);  // completed before the projection
  const int g = lane / LPV;
  const int l = lane % LPV;
  const int64_t row = one_vec ? (wib == 0 && g == 0 ? vblock : n) : (vblock * (kRotThreads / 32) + wib) * VPW + g;
  const bool valid = row < n;

  float v[KCH][4];
#pragma unroll
  for (int k = 0; k < KCH; ++k) {
    const int j0 = 4 * (l + LPV * k);
    if (valid) {
      if (dtype == TQ_F32) {
        const float4 t = *reinterpret_cast<const float4 *>(static_cast<const float *>(x) + row * ld + j0);
        v[k][0] = t.x; v[k][1] = t.y; v[k][2] = t.z; v[k][3] = t.w;
      } else {
        const uint2 t = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(x) + row * ld + j0);
        v[k][0] = __uint_as_float(t.x << 16);
        v[k][1] = __uint_as_float(t.x & 0xffff0000u);
        v[k][2] = __uint_as_float(t.y << 16);
        v[k][3] = __uint_as_float(t.y & 0xffff0000u);
      }
    } else {
      v[k][0] = v[k][1] = v[k][2] = v[k][3] = 0.f;
    }
  }

  // ||x|| and the unit vector (encode only; queries are rotated as they are)
  float nu = 0.f, inv = 1.f;
  if (mode == ROT_ENCODE) {
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < KCH; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) ss = fmaf(v[k][e], v[k][e], ss);
    ss = group_sum<LPV>(ss);
    nu = sqrtf(ss);
    inv = nu > 0.f ? 1.f / nu : 0.f;
  }
  // D (random signs) and the unit scaling
#pragma unroll
  for (int k = 0; k < KCH; ++k) {
    const float4 sg = *reinterpret_cast<const float4 *>(c.signs + 4 * (l + LPV * k));
    v[k][0] *= inv * sg.x; v[k][1] *= inv * sg.y; v[k][2] *= inv * sg.z; v[k][3] *= inv * sg.w;
  }
  // Walsh-Hadamard butterflies
  fwht_lanes<D>(v, l);
#pragma unroll
  for (int k = 0; k < KCH; ++k)
#pragma unroll
    for (int e = 0; e < 4; ++e) v[k][e] *= c.inv_sqrt_d;

  if (mode == ROT_QUERY) {
    if (valid)
#pragma unroll
      for (int k = 0; k < KCH; ++k)
        *reinterpret_cast<float4 *>(resid + row * D + 4 * (l + LPV * k)) =
            make_float4(v[k][0], v[k][1], v[k][2], v[k][3]);
    return;
  }

  // Lloyd-Max codes (count of thresholds <= y) and the residual
  int code[KCH][4];
  float rr = 0.f;
#pragma unroll
  for (int k = 0; k < KCH; ++k)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float y = v[k][e];
      int q = 0;
      float cc = c.centroids[0];
      for (int i = 0; i < c.levels - 1; ++i) {
        const bool ge = y >= c.thresholds[i];
        q += ge ? 1 : 0;
        cc = ge ? c.centroids[i + 1] : cc;
      }
      code[k][e] = q;
      v[k][e] = y - cc;  // residual
      rr = fmaf(v[k][e], v[k][e], rr);
    }

  const int64_t slot = valid ? (slots ? slots[row] : row) : -1;
  const bool store = valid && slot >= 0 && slot < capacity;

  if (c.layout == TQ_LAYOUT_BLOCK16) {
    // token-transposed blocks: set this slot's bit in the shared words of its 16-slot block
    if (store) {
      uint32_t *blk = codes + (slot >> 4) * (int64_t)(16 * c.code_words);
      const int tok = (int)(slot & 15);
#pragma unroll
      for (int k = 0; k < KCH; ++k)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * (l + LPV * k) + e;
          const int cd = code[k][e];
          for (int q = 0; q < c.bits / 2; ++q) {
            const uint32_t mask = (1u << tok) | (1u << (16 + tok));
            const uint32_t val = ((uint32_t)((cd >> (2 * q)) & 1) << tok) |
                                 ((uint32_t)((cd >> (2 * q + 1)) & 1) << (16 + tok));
            atomicAnd(&blk[q * D + j], ~mask);
            atomicOr(&blk[q * D + j], val);
          }
          if (c.bits & 1) {
            const int sh = 16 * (j & 1) + tok;
            uint32_t *w = &blk[(c.bits / 2) * D + (j >> 1)];
            atomicAnd(w, ~(1u << sh));
            atomicOr(w, (uint32_t)((cd >> (c.bits - 1)) & 1) << sh);
          }
        }
      if (l == 0) st_norm(norm, slot, nu, c.norm16);
    }
    if (staged) stage_async_wait();  // no copy may be left in flight
    return;  // MSE-only: no residual
  }

  // pack the bit-planes
  uint32_t *st = stage[wib][g];
  for (int i = l; i < c.code_words; i += LPV) st[i] = 0u;
  __syncwarp();
  for (int t = 0; t < c.bits; ++t)
#pragma unroll
    for (int k = 0; k < KCH; ++k) {
      uint32_t nib = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) nib |= (uint32_t)((code[k][e] >> t) & 1) << e;
      const int pos = t * D + 4 * (l + LPV * k);
      atomicOr(&st[pos >> 5], nib << (pos & 31));
    }
  __syncwarp();

  if (store) {
    uint4 *dst = reinterpret_cast<uint4 *>(codes + slot * c.code_words);
    for (int i = l; i < c.code_words / 4; i += LPV)
      dst[i] = make_uint4(st[4 * i], st[4 * i + 1], st[4 * i + 2], st[4 * i + 3]);
    if (l == 0) st_norm(norm, slot, nu, c.norm16);
  }
  if (c.srht && fsigns != nullptr) {
    // structured QJL ("TurboQuant 学习路径" 二.2, fast JL y = P H D x): z = H (D2 r), the first m
    // coordinates' signs, by the same butterflies as the rotation (no projection matrix)
    const float gamma = sqrtf(group_sum<LPV>(rr));
    if (store && l == 0) st_norm(rnorm, slot, gamma, c.norm16);
#pragma unroll
    for (int k = 0; k < KCH; ++k) {
      const float4 sg = *reinterpret_cast<const float4 *>(c.qjl_signs + 4 * (l + LPV * k));
      v[k][0] *= sg.x; v[k][1] *= sg.y; v[k][2] *= sg.z; v[k][3] *= sg.w;
    }
    fwht_lanes<D>(v, l);
    __syncwarp();  // the staging words were read by the code store above
    for (int i = l; i < c.sign_words; i += LPV) st[i] = 0u;
    __syncwarp();
#pragma unroll
    for (int k = 0; k < KCH; ++k) {
      const int j0 = 4 * (l + LPV * k);
      if (j0 < c.m) {
        uint32_t nib = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) nib |= (v[k][e] >= 0.f ? 1u : 0u) << e;
        atomicOr(&st[j0 >> 5], nib << (j0 & 31));
      }
    }
    __syncwarp();
    if (store) {
      uint4 *dst = reinterpret_cast<uint4 *>(fsigns + slot * c.sign_words);
      for (int i = l; i < c.sign_words / 4; i += LPV)
        dst[i] = make_uint4(st[4 * i], st[4 * i + 1], st[4 * i + 2], st[4 * i + 3]);
    }
    return;
  }
  if constexpr (D >= 128) {
    if (fsigns != nullptr) {
      // fused QJL projection for small batches: one vector per warp, z_i = <S_i, r> with the
      // residual broadcast from shared memory, lane = output row within each group of 32
      if (staged) {
        stage_async_wait();
        __syncthreads();
      }
      const float gamma = sqrtf(group_sum<LPV>(rr));
      if (store && l == 0) st_norm(rnorm, slot, gamma, c.norm16);
      float *rb = rbuf[one_vec ? 0 : wib];
      if (!one_vec || wib == 0)
#pragma unroll
        for (int k = 0; k < KCH; ++k)
#pragma unroll
          for (int e = 0; e < 4; ++e) rb[4 * (l + LPV * k) + e] = v[k][e];
      if (one_vec) {
        __shared__ int64_t oslot;
        __shared__ int ostore;
        if (threadIdx.x == 0) {
          oslot = slot;
          ostore = store ? 1 : 0;
        }
        __syncthreads();
        if (wib < c.m / 32) {
          const int w = wib;
          float z = 0.f;
          if (staged) {
            const float4 *Srow = reinterpret_cast<const float4 *>(sS + (32 * w + lane) * (D + 4));
#pragma unroll 8
            for (int j4 = 0; j4 < D / 4; ++j4) {
              const float4 sv = Srow[j4];
              z = fmaf(sv.x, rb[4 * j4], z);
              z = fmaf(sv.y, rb[4 * j4 + 1], z);
              z = fmaf(sv.z, rb[4 * j4 + 2], z);
              z = fmaf(sv.w, rb[4 * j4 + 3], z);
            }
          } else {
            // S transposed: the warp reads 32 consecutive floats per coordinate (same order of sums)
            const float *Sc = c.St + 32 * w + lane;
#pragma unroll 32
            for (int j = 0; j < D; ++j) z = fmaf(Sc[(int64_t)j * c.m], rb[j], z);
          }
          const unsigned bal = __ballot_sync(TQ_FULL_MASK, z >= 0.f);
          if (ostore && lane == 0) fsigns[oslot * c.sign_words + w] = bal;
        }
        return;
      }
      __syncwarp();
      for (int w = 0; w < c.m / 32; ++w) {
        float z = 0.f;
        if (staged) {
          const float4 *Srow = reinterpret_cast<const float4 *>(sS + (32 * w + lane) * (D + 4));
#pragma unroll 8
          for (int j4 = 0; j4 < D / 4; ++j4) {
            const float4 sv = Srow[j4];
            z = fmaf(sv.x, rb[4 * j4], z);
            z = fmaf(sv.y, rb[4 * j4 + 1], z);
            z = fmaf(sv.z, rb[4 * j4 + 2], z);
            z = fmaf(sv.w, rb[4 * j4 + 3], z);
          }
        } else {
          const float *Sc = c.St + 32 * w + lane;
#pragma unroll 32
          for (int j = 0; j < D; ++j) z = fmaf(Sc[(int64_t)j * c.m], rb[j], z);
        }
        const unsigned bal = __ballot_sync(TQ_FULL_MASK, z >= 0.f);
        if (store && lane == 0) fsigns[slot * c.sign_words + w] = bal;
      }
      return;
    }
  }
  if (resid != nullptr) {
    const float gamma = sqrtf(group_sum<LPV>(rr));
    if (store && l == 0) st_norm(rnorm, slot, gamma, c.norm16);
    if (valid)
#pragma unroll
      for (int k = 0; k < KCH; ++k)
        *reinterpret_cast<float4 *>(resid + row * D + 4 * (l + LPV * k)) =
            make_float4(v[k][0], v[k][1], v[k][2], v[k][3]);
  }
}

