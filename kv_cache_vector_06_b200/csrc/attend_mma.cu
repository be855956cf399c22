// Tensor-core decode attention for head_dim 128 and 4 query heads per KV head.
//
// Same mathematics as attend_split_kernel (estimated logits "谷歌 TurboQuant 深度拆解" 第二部分
// 第二步, softmax, value sum in the rotated domain), reorganised so that the per-bit work runs on
// the tensor cores as exact integer matrix products:
//
//  * A symmetric Lloyd-Max codebook is an odd function of the bit-plane signs s_P = 2 b_P - 1:
//      c(code) = sum_P e_P s_P  (+ e_3 s_0 s_1 s_2 for 3 bits),
//    so <q', c[code]> = sum_P 2 e_P <q', b_P> - (sum_P e_P) sum_j q'_j, with b_P the 0/1 plane
//    (the 3-bit cubic term uses the parity plane b_0 ^ b_1 ^ b_2).  The QJL term is likewise
//    2 <p, b_sign> - sum_i p_i.
//  * Logits: one m16n8k32 u8 x s8 MMA per (16 keys, plane, 32 coordinates).  A = the keys' bit
//    words masked in place (w & (0x01010101 << shift): bytes 0 or 2^shift, one LOP3 per 4
//    elements); B = the query term 2 e_P q' (or 2 p) in 32-bit fixed point split into four signed
//    byte limbs and pre-scaled by 2^-shift, built once per (sequence, KV head) by kfrag_kernel.
//    Columns: 4 heads x 4 limbs (two n-tiles), so each thread ends with all limbs of one head.
//  * Values are stored token-transposed (TQ_LAYOUT_BLOCK16): one 32-bit word = one coordinate of
//    16 tokens in two planes, so (w >> t) & 0x01010101 gives four tokens of one coordinate, the
//    A operand of an MMA that contracts over tokens.  B = the softmax weights times the value
//    norms in unsigned 16-bit fixed point (two byte limbs) relative to the chunk's largest one,
//    rounded with a deterministic dither so that the many sub-unit weights of a long tail are
//    unbiased rather than all rounded down; columns = 4 heads x 2 planes x 2 limbs.  The
//    codebook's constant term uses the same integer weights as the MMA.
//  * Softmax is two-pass per chunk (all logits of the chunk, then one max per head), so every
//    value product of the chunk shares one fixed-point scale and the int32 accumulators need no
//    rescaling; splits are merged by attend_combine_kernel as for the general kernel.
// Each CTA: 8 warps, one chunk of CH tokens of one (sequence, KV head).
#include <cmath>

#include "device_common.cuh"
#include "rotate_device.cuh"

namespace {

constexpr int kD = 128;
constexpr int kG = 4;

// Poll count of the test hook's bounded wait (0 = off); see tq_debug_wait_probe.
__device__ int g_tq_wait_probe;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct MmaArgs {
  int hq, hkv, max_len, chunk, splits, block_size, max_blocks;
  int64_t ctx_stride;
  float scale;
  const int32_t *seq_lens;
  const int32_t *block_table;
  tq_packed k, v;
  int *counter;  // per (sequence, KV head): CTAs done (zeroed by the query-fragment kernel)
  float *out;    // final output when the kernel merges its splits itself, else null
};

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_u8u8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Uniform value in [0, 1) from a 32-bit key: the fractional part of key * (golden ratio), a
// low-discrepancy sequence over consecutive keys (deterministic dither for rounding).
__device__ __forceinline__ float dither(uint32_t x) {
  // top 23 bits of the product as the mantissa of a float in [1, 2), minus 1 (no conversion unit)
  return __uint_as_float(0x3F800000u | ((x * 2654435769u) >> 9)) - 1.0f;
}

// floor(v) for 0 <= v < 2^23, as the low mantissa bits of 2^23 + floor(v): a round-down add on the
// FMA pipe instead of a float-to-integer conversion.  The result's bytes 0 and 1 are floor(v)'s.
__device__ __forceinline__ uint32_t floor_bits(float v) { return __float_as_uint(__fadd_rd(v, 8388608.f)); }

__device__ __forceinline__ int64_t token_slot(const MmaArgs &a, int b, int h, int t) {
  if (a.block_table) {
    const int blk = a.block_table[(int64_t)b * a.max_blocks + t / a.block_size];
    return blk < 0 ? -1 : ((int64_t)blk * a.hkv + h) * a.block_size + t % a.block_size;
  }
  return ((int64_t)b * a.hkv + h) * a.ctx_stride + t;
}

__device__ __forceinline__ float warp_max_f(float x) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) x = fmaxf(x, __shfl_xor_sync(TQ_FULL_MASK, x, s));
  return x;
}
__device__ __forceinline__ float warp_sum_f(float x) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) x += __shfl_xor_sync(TQ_FULL_MASK, x, s);
  return x;
}

template <int BK, bool QJL>
struct KPlanes {
  static constexpr int code = BK + (BK == 3 ? 1 : 0);  // code planes (+ parity plane for 3 bits)
  static constexpr int all = code + (QJL ? 1 : 0);     // + the QJL sign plane
  static constexpr int regs = all * 4 * 2 * 2;          // planes x k-steps x n-tiles x registers
};

// Query-side B fragments of the logit MMAs for one (sequence, KV head): for plane P, k-step s,
// n-tile nt, register r and lane (gid, t): bytes i = 0..3 hold limb (gid & 1) + 2 nt of
//   round(X_P[head gid/2][32 t + s + 4 r + 8 i] * 2^(F - s - 4 r)),
// X_P = 2 e_P q' (code planes, parity), 2 p (sign plane); F per head and part so that
// |X| 2^F <= 2^30.  kconst: 2^-F_code, 2^-F_sign, (sum e_P) sum q', sum p per head.
template <int BK, bool QJL>
__device__ __forceinline__ void kfrag_group(const TqConsts &kc, const void *__restrict__ q, int dtype,
                                            uint32_t *__restrict__ kfrag, float *__restrict__ kconst,
                                            int *__restrict__ counter, int grp, float *sS) {
  using KP = KPlanes<BK, QJL>;
  __shared__ float qs[kG][kD];           // q', the rotated queries
  __shared__ float X[KP::all][kG][kD];
  __shared__ float red[kG][4];
  __shared__ int fexp[kG][2];
  // grp = b * hkv + h; its query heads are rows grp * 4 + g
  const int tid = threadIdx.x;
  // S (for p = S q') is copied asynchronously while q' is formed
  if constexpr (QJL) stage_rows_padded_async(sS, kc.S, kD, kD);
  // q' = (1/sqrt d) H (D q): load with the signs applied, then the butterflies in shared memory
  for (int i = tid; i < kG * kD; i += kThreads) {
    const int g = i / kD, j = i % kD;
    const int64_t o = ((int64_t)grp * kG + g) * kD + j;
    const float x = dtype == TQ_F32 ? static_cast<const float *>(q)[o]
                                    : bf16_to_f32(static_cast<const uint16_t *>(q)[o]);
    qs[g][j] = x * kc.signs[j];
  }
  __syncthreads();
  for (int hh = 1; hh < kD; hh <<= 1) {
    const int g = tid >> 6, i = tid & 63;  // 4 heads x 64 butterflies = 256 threads
    const int lo = (i / hh) * 2 * hh + (i % hh);
    const float a0 = qs[g][lo], b0 = qs[g][lo + hh];
    __syncthreads();
    qs[g][lo] = a0 + b0;
    qs[g][lo + hh] = a0 - b0;
    __syncthreads();
  }
  for (int i = tid; i < kG * kD; i += kThreads) {
    const int g = i / kD, j = i % kD;
    const float qv = qs[g][j] * kc.inv_sqrt_d;
    qs[g][j] = qv;
#pragma unroll
    for (int P = 0; P < BK; ++P) X[P][g][j] = 2.f * kc.plane_coef[P] * qv;
    if constexpr (BK == 3) X[3][g][j] = 2.f * kc.plane_coef[3] * qv;
  }
  __syncthreads();
  if constexpr (QJL) {
    // p = S q' for the 4 heads: S staged in shared memory (row stride kD + 4), thread (row i,
    // head pair) dots row i with two q'
    stage_async_wait();
    __syncthreads();
    const int i = tid & (kD - 1), gp = tid >> 7;
    const float4 *Srow = reinterpret_cast<const float4 *>(sS + i * (kD + 4));
    float p0 = 0.f, p1 = 0.f;
#pragma unroll 8
    for (int j4 = 0; j4 < kD / 4; ++j4) {
      const float4 sv = Srow[j4];
      p0 = fmaf(sv.x, qs[2 * gp][4 * j4], p0);
      p0 = fmaf(sv.y, qs[2 * gp][4 * j4 + 1], p0);
      p0 = fmaf(sv.z, qs[2 * gp][4 * j4 + 2], p0);
      p0 = fmaf(sv.w, qs[2 * gp][4 * j4 + 3], p0);
      p1 = fmaf(sv.x, qs[2 * gp + 1][4 * j4], p1);
      p1 = fmaf(sv.y, qs[2 * gp + 1][4 * j4 + 1], p1);
      p1 = fmaf(sv.z, qs[2 * gp + 1][4 * j4 + 2], p1);
      p1 = fmaf(sv.w, qs[2 * gp + 1][4 * j4 + 3], p1);
    }
    X[KP::code][2 * gp][i] = 2.f * p0;
    X[KP::code][2 * gp + 1][i] = 2.f * p1;
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  if (warp < kG) {
    const int g = warp;
    float mc = 0.f, ms = 0.f, sq = 0.f, sp = 0.f;
    for (int j = lane; j < kD; j += 32) {
#pragma unroll
      for (int P = 0; P < KP::code; ++P) mc = fmaxf(mc, fabsf(X[P][g][j]));
      if constexpr (QJL) {
        ms = fmaxf(ms, fabsf(X[KP::code][g][j]));
        sp += 0.5f * X[KP::code][g][j];
      }
      sq += qs[g][j];
    }
    mc = warp_max_f(mc);
    ms = warp_max_f(ms);
    sq = warp_sum_f(sq);
    sp = warp_sum_f(sp);
    if (lane == 0) {
      int ec = 0, es = 0;
      frexpf(mc, &ec);  // mc < 2^ec
      frexpf(ms, &es);
      // |X| 2^F <= 2^30: four signed byte limbs
      fexp[g][0] = mc > 0.f ? 30 - ec : 0;
      fexp[g][1] = ms > 0.f ? 30 - es : 0;
      red[g][0] = pow2i(-fexp[g][0]);
      red[g][1] = pow2i(-fexp[g][1]);
      red[g][2] = kc.plane_coef_sum * sq;
      red[g][3] = sp;
    }
  }
  __syncthreads();
  if (tid < 16) kconst[(int64_t)grp * 16 + tid] = red[tid % 4][tid / 4];
  if (tid == 0) counter[grp] = 0;  // the split kernel that follows counts its finished CTAs here
  uint32_t *out = kfrag + (int64_t)grp * KP::regs * 32;
  // layout [plane][k-step][lane][n-tile, register]: one 16-byte load per lane and k-step.
  // Balanced byte limbs: with w = v + 0x80808080 (mod 2^32), limb k of v = byte k of w - 128,
  // stored as its two's-complement byte, byte k of w ^ 0x80.
  for (int idx = tid; idx < KP::regs * 32; idx += kThreads) {
    const int r = idx & 1;
    const int nt = (idx >> 1) & 1;
    const int ln = (idx >> 2) & 31;
    const int s = (idx >> 7) & 3;
    const int P = idx >> 9;
    const int gid = ln >> 2, t = ln & 3;
    const int g = gid >> 1, limb = (gid & 1) + 2 * nt;
    const float sc = pow2i(fexp[g][(QJL && P == KP::code) ? 1 : 0] - s - 4 * r);
    const uint32_t sel = (uint32_t)limb | ((uint32_t)(4 + limb) << 4);  // byte `limb` of two words
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = (uint32_t)__float2int_rn(X[P][g][32 * t + s + 4 * r + 8 * i] * sc) + 0x80808080u;
    out[idx] = __byte_perm(__byte_perm(w[0], w[1], sel), __byte_perm(w[2], w[3], sel), 0x5410) ^ 0x80808080u;
  }
}

// kfrag_group's work for one query head g of the group: the same arithmetic in the same order
// (so the fragments are bit-identical), a quarter of the work per block.
template <int BK, bool QJL>
__device__ __forceinline__ void kfrag_head(const TqConsts &kc, const void *__restrict__ q, int dtype,
                                           uint32_t *__restrict__ kfrag, float *__restrict__ kconst,
                                           int *__restrict__ counter, int grp, int g, float *sS) {
  using KP = KPlanes<BK, QJL>;
  __shared__ float qs[kD];
  __shared__ float X[KP::all][kD];
  __shared__ float red[4];
  __shared__ int fexp[2];
  const int tid = threadIdx.x;
  if constexpr (QJL) stage_rows_padded_async(sS, kc.S, kD, kD);
  for (int j = tid; j < kD; j += kThreads) {
    const int64_t o = ((int64_t)grp * kG + g) * kD + j;
    const float x = dtype == TQ_F32 ? static_cast<const float *>(q)[o]
                                    : bf16_to_f32(static_cast<const uint16_t *>(q)[o]);
    qs[j] = x * kc.signs[j];
  }
  __syncthreads();
  for (int hh = 1; hh < kD; hh <<= 1) {
    const int i = tid & 63;  // 64 butterflies (threads 64.. repeat them harmlessly: same values)
    const int lo = (i / hh) * 2 * hh + (i % hh);
    const float a0 = qs[lo], b0 = qs[lo + hh];
    __syncthreads();
    if (tid < 64) {
      qs[lo] = a0 + b0;
      qs[lo + hh] = a0 - b0;
    }
    __syncthreads();
  }
  for (int j = tid; j < kD; j += kThreads) {
    const float qv = qs[j] * kc.inv_sqrt_d;
    qs[j] = qv;
#pragma unroll
    for (int P = 0; P < BK; ++P) X[P][j] = 2.f * kc.plane_coef[P] * qv;
    if constexpr (BK == 3) X[3][j] = 2.f * kc.plane_coef[3] * qv;
  }
  __syncthreads();
  if constexpr (QJL) {
    stage_async_wait();
    __syncthreads();
    if (tid < kD) {
      const float4 *Srow = reinterpret_cast<const float4 *>(sS + tid * (kD + 4));
      float p0 = 0.f;
#pragma unroll 8
      for (int j4 = 0; j4 < kD / 4; ++j4) {
        const float4 sv = Srow[j4];
        p0 = fmaf(sv.x, qs[4 * j4], p0);
        p0 = fmaf(sv.y, qs[4 * j4 + 1], p0);
        p0 = fmaf(sv.z, qs[4 * j4 + 2], p0);
        p0 = fmaf(sv.w, qs[4 * j4 + 3], p0);
      }
      X[KP::code][tid] = 2.f * p0;
    }
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    float mc = 0.f, ms = 0.f, sq = 0.f, sp = 0.f;
    for (int j = lane; j < kD; j += 32) {
#pragma unroll
      for (int P = 0; P < KP::code; ++P) mc = fmaxf(mc, fabsf(X[P][j]));
      if constexpr (QJL) {
        ms = fmaxf(ms, fabsf(X[KP::code][j]));
        sp += 0.5f * X[KP::code][j];
      }
      sq += qs[j];
    }
    mc = warp_max_f(mc);
    ms = warp_max_f(ms);
    sq = warp_sum_f(sq);
    sp = warp_sum_f(sp);
    if (lane == 0) {
      int ec = 0, es = 0;
      frexpf(mc, &ec);
      frexpf(ms, &es);
      fexp[0] = mc > 0.f ? 30 - ec : 0;
      fexp[1] = ms > 0.f ? 30 - es : 0;
      red[0] = pow2i(-fexp[0]);
      red[1] = pow2i(-fexp[1]);
      red[2] = kc.plane_coef_sum * sq;
      red[3] = sp;
    }
  }
  __syncthreads();
  if (tid < 4) kconst[(int64_t)grp * 16 + 4 * tid + g] = red[tid];
  if (g == 0 && tid == 0) counter[grp] = 0;  // the split kernel that follows counts its CTAs here
  // this head's fragment words: lanes 8 g .. 8 g + 7 of every (plane, k-step, n-tile, register)
  uint32_t *out = kfrag + (int64_t)grp * KP::regs * 32;
  for (int w = tid; w < KP::regs * 8; w += kThreads) {
    const int r = w & 1, nt = (w >> 1) & 1, ls = (w >> 2) & 7, st = (w >> 5) & 3, P = w >> 7;
    const int ln = 8 * g + ls;
    const int t = ln & 3, limb = ((ln >> 2) & 1) + 2 * nt;
    const float sc = pow2i(fexp[(QJL && P == KP::code) ? 1 : 0] - st - 4 * r);
    const uint32_t sel = (uint32_t)limb | ((uint32_t)(4 + limb) << 4);
    uint32_t wv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) wv[i] = (uint32_t)__float2int_rn(X[P][32 * t + st + 4 * r + 8 * i] * sc) + 0x80808080u;
    out[(((P * 4 + st) * 32 + ln) * 2 + nt) * 2 + r] =
        __byte_perm(__byte_perm(wv[0], wv[1], sel), __byte_perm(wv[2], wv[3], sel), 0x5410) ^ 0x80808080u;
  }
}

template <int BK, bool QJL>
__global__ void __launch_bounds__(kThreads)
kfrag_kernel(TqConsts kc, const void *__restrict__ q, int dtype, uint32_t *__restrict__ kfrag,
             float *__restrict__ kconst, int *__restrict__ counter) {
  extern __shared__ __align__(16) float sS[];
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");  // the attention grid may start
  kfrag_group<BK, QJL>(kc, q, dtype, kfrag, kconst, counter, blockIdx.x, sS);
}

// One launch for the work that precedes the split kernel in a decode step: blocks
// [0, nkb) append-encode the new keys (one per block with QJL, whose projection four warps share;
// else 8 per block), blocks [nkb, nkb + nvb) the new values (8 per block), and the remaining
// blocks build one query head's fragments each.  The jobs are independent, so their latencies
// overlap instead of adding up.
template <int BK, bool QJL>
__global__ void __launch_bounds__(kThreads)
decode_prep_kernel(TqConsts kc, TqConsts vc, const void *__restrict__ knew, const void *__restrict__ vnew,
                   int kvdtype, int64_t nnew, const int64_t *__restrict__ slots, tq_packed kp, tq_packed vp,
                   const void *__restrict__ q, int qdtype, uint32_t *__restrict__ kfrag,
                   float *__restrict__ kconst, int *__restrict__ counter, int nkb, int nvb) {
  extern __shared__ __align__(16) float sS[];
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");  // the attention grid may start
  const int bid = blockIdx.x;
  if (bid < nkb) {
    // keys: with QJL one row per block (warps 0-3 share its projection), else 8 rows per block
    rotate_rows<kD>(kc, ROT_ENCODE, knew, kvdtype, nnew, kD, slots, kp.capacity, static_cast<uint32_t *>(kp.codes),
                    kp.norm, kp.rnorm, nullptr, QJL ? static_cast<uint32_t *>(kp.signs) : nullptr, bid, sS, QJL);
  } else if (bid < nkb + nvb) {
    rotate_rows<kD>(vc, ROT_ENCODE, vnew, kvdtype, nnew, kD, slots, vp.capacity, static_cast<uint32_t *>(vp.codes),
                    vp.norm, nullptr, nullptr, nullptr, bid - nkb, sS);
  } else {
    const int qh = bid - nkb - nvb;  // query head: group qh / 4, head qh % 4
    kfrag_head<BK, QJL>(kc, q, qdtype, kfrag, kconst, counter, qh / kG, qh % kG, sS);
  }
}

// Fixed-point scale of a sub-chunk's value weights: with top = max W * 2 max_P e_P, the integer
// weights floor(W 2 e_P sc + dither) stay below 2^16.  Returns sc and 1 / (128 sc).
__device__ __forceinline__ void weight_scale(float top, float &sc, float &inv128) {
  if (!(top > 0.f)) {
    sc = 1.f;
    inv128 = 1.f / 128.f;
    return;
  }
  int e = ((__float_as_int(top) >> 23) & 0xff) - 126;  // top < 2^e
  e = e < -110 ? -110 : (e > 126 ? 126 : e);
  sc = pow2i(16 - e) * (1.f - 1.f / 512.f);
  inv128 = pow2i(e - 23) * (512.f / 511.f);
}
// Largest of the 8 per-warp partials of one head.
__device__ __forceinline__ float max8(const float *p) {
  const float4 u = *reinterpret_cast<const float4 *>(p), v = *reinterpret_cast<const float4 *>(p + 4);
  return fmaxf(fmaxf(fmaxf(u.x, u.y), fmaxf(u.z, u.w)), fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
}

// 32-bit multiply kept as such (an opaque multiplier: a power of two here, which would otherwise
// become a shift on the integer ALU pipe).
__device__ __forceinline__ uint32_t mul_lo(uint32_t x, uint32_t m) {
  uint32_t r;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(m));
  return r;
}

constexpr int kSub = 256;          // tokens per sub-chunk (one staging buffer)
constexpr int kSubBlk = kSub / 16;  // 16-token blocks per sub-chunk
constexpr int kLgS = kSub + 8;      // row stride of the logit/weight array (bank-conflict padding)

// Shared-memory carve-up of attend_mma_kernel (bytes): two staging buffers (the sub-chunk being
// computed and the one being loaded), then the per-sub-chunk work arrays.
template <int BK, int BV, bool QJL>
struct MmaSmem {
  static constexpr int NB = kSubBlk;
  static constexpr int KCW = BK * 4;            // K code words per key
  static constexpr int KSW = QJL ? 4 : 0;       // K sign words per key
  static constexpr int VBW = BV * kD / 2;       // V words per 16-token block
  static constexpr int X1W = BV == 3 ? kD : 0;  // (plane 2, parity) words per block
  // offsets inside one staging buffer
  static constexpr size_t kc = 0;
  static constexpr size_t ks = kc + (size_t)kSub * KCW * 4;
  static constexpr size_t kn = ks + (size_t)kSub * KSW * 4;
  static constexpr size_t kr = kn + (size_t)kSub * 4;
  static constexpr size_t vc = kr + (size_t)kSub * 4;
  static constexpr size_t vn = vc + (size_t)NB * VBW * 4;
  static constexpr size_t buf = vn + (size_t)kSub * 4;
  // work arrays
  static constexpr size_t x1 = 2 * buf;
  static constexpr size_t lg = x1 + (size_t)NB * X1W * 4;
  static constexpr size_t vf = lg + (size_t)kG * kLgS * 4;
  static constexpr size_t kf = vf + (size_t)NB * 32 * 16;
  static constexpr size_t vb = kf + (size_t)KPlanes<BK, QJL>::regs * 32 * 4;
  static constexpr int MAXBLK = 64;  // blocks per CTA at most (a.chunk <= 1024 tokens)
  static constexpr size_t st = vb + (size_t)MAXBLK * 8;
  static constexpr size_t pw = st + 16 * kG * 4;  // per-warp partials (max logit, sum w, sum X, max ||v||)
  static constexpr size_t br = pw + 4 * kG * kWarps * 4;  // two mbarriers, one per staging buffer
  static constexpr size_t total = br + 48;  // + flags at br + 16, merge barrier at br + 32
  static_assert((size_t)4 * kG * kD * 4 <= 2 * buf, "the value-sum buffer reuses the staging buffers");
  static_assert(buf % 16 == 0 && x1 % 16 == 0 && kf % 16 == 0, "16-byte aligned regions");
};

// The arrays a sub-chunk is copied from, one bulk copy (or one per block when paged) each.
template <bool QJL>
struct StageArrays {
  static constexpr int n = QJL ? 6 : 4;  // K codes, V codes, ||k||, ||v|| (+ K signs, gamma)
};

// Array `arr` of a sub-chunk copy: source base, offset in the staging buffer, bytes per 16-slot
// block and source bytes per slot.  (V codes are addressed by block: slot / 16 * block bytes ==
// slot * (block bytes / 16).)
template <int BK, int BV, bool QJL>
__device__ __forceinline__ void stage_array(const MmaArgs &a, int arr, const char *&src, size_t &doff, unsigned &per,
                                            int64_t &sstride) {
  using SM = MmaSmem<BK, BV, QJL>;
  switch (arr) {
    case 0: src = static_cast<const char *>(a.k.codes); doff = SM::kc; per = 16 * SM::KCW * 4; sstride = SM::KCW * 4; break;
    case 1: src = static_cast<const char *>(a.v.codes); doff = SM::vc; per = SM::VBW * 4; sstride = SM::VBW * 4 / 16; break;
    case 2: src = reinterpret_cast<const char *>(a.k.norm); doff = SM::kn; per = 64; sstride = 4; break;
    case 3: src = reinterpret_cast<const char *>(a.v.norm); doff = SM::vn; per = 64; sstride = 4; break;
    case 4: src = static_cast<const char *>(a.k.signs); doff = SM::ks; per = 256; sstride = 16; break;
    default: src = reinterpret_cast<const char *>(a.k.rnorm); doff = SM::kr; per = 64; sstride = 4; break;
  }
}

// Issue the bulk copies of sub-chunk `sc` of the CTA (blocks [16 sc, 16 sc + 16) of its range)
// into staging buffer `sb`, completing on `bar` (initialised with one arrival per array).  Warp
// `arr` (< StageArrays::n) copies array `arr`.  vb[k] = first slot of the CTA's block k, or -1
// (resolved once per CTA); nlead = number of leading valid blocks of the CTA (contiguous layout,
// where they are one run of consecutive slots: one copy per array); paged: one copy per block.
// `extra` bytes (landing on the same barrier, issued by the caller after this returns) are
// expected by warp 0.
template <int BK, int BV, bool QJL>
__device__ __forceinline__ void stage_sub(const MmaArgs &a, int sc, const int64_t *vb, int nlead,
                                          unsigned char *sb, uint64_t *bar, unsigned extra) {
  using SM = MmaSmem<BK, BV, QJL>;
  const int arr = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const char *src;
  size_t doff;
  unsigned per;
  int64_t sstride;
  stage_array<BK, BV, QJL>(a, arr, src, doff, per, sstride);
  const int k0 = SM::NB * sc;
  if (!a.block_table) {
    if (lane == 0) {
      int n = nlead - k0;
      n = n < 0 ? 0 : (n > SM::NB ? SM::NB : n);
      mbar_expect_arrive(bar, per * (unsigned)n + (arr == 0 ? extra : 0u));
      if (n > 0) bulk_g2s(sb + doff, src + vb[k0] * sstride, per * (unsigned)n, bar);
    }
  } else {
    const int64_t base = lane < SM::NB ? vb[k0 + lane] : -1;
    const unsigned valid = __ballot_sync(TQ_FULL_MASK, base >= 0);
    if (lane == 0) mbar_expect_arrive(bar, per * (unsigned)__popc(valid) + (arr == 0 ? extra : 0u));
    __syncwarp();
    if (base >= 0) bulk_g2s(sb + doff + (size_t)lane * per, src + base * sstride, per, bar);
  }
}

// One CTA = one (sequence, KV head) and a contiguous range of a.chunk tokens (a multiple of 16),
// streamed in sub-chunks of kSub tokens: the next sub-chunk's bulk copies are in flight while
// the current one is computed.  Softmax runs across sub-chunks with a running maximum: the value
// sums of each sub-chunk use that sub-chunk's own fixed-point scale and are folded into fp32
// accumulators rescaled by e^{M_old - M_new}.
template <int BK, int BV, bool QJL>
__global__ void __launch_bounds__(kThreads, 2)
attend_mma_kernel(TqConsts kc, TqConsts vc, MmaArgs a, const uint32_t *__restrict__ kfrag,
                  const float *__restrict__ kconst, float *__restrict__ part) {
  using KP = KPlanes<BK, QJL>;
  using SM = MmaSmem<BK, BV, QJL>;
  constexpr int NB = SM::NB;
  constexpr int VT = BV == 3 ? 2 : 1;  // value word types: (p0,p1) and (p2, parity)
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t *sx1 = reinterpret_cast<uint32_t *>(smem + SM::x1);
  float *lg = reinterpret_cast<float *>(smem + SM::lg);          // [kG][kLgS] logits, then weights
  uint4 *vfrag = reinterpret_cast<uint4 *>(smem + SM::vf);       // [NB][32]
  const uint4 *kf4 = reinterpret_cast<const uint4 *>(smem + SM::kf);  // [plane][k-step][32]
  int64_t *vball = reinterpret_cast<int64_t *>(smem + SM::vb);   // [MAXBLK] first slot of each block
  float *hM = reinterpret_cast<float *>(smem + SM::st);          // running max per head
  float *hL = hM + kG;                                           // running sum of e^{l - M}
  float *pmax = reinterpret_cast<float *>(smem + SM::pw);        // [kG][kWarps] max logit
  float *psw = pmax + kG * kWarps;                               // [kG][kWarps] sum of w
  int *pcs = reinterpret_cast<int *>(psw + kG * kWarps);         // [kG][kWarps] sum of integer weights
  float *pnv = reinterpret_cast<float *>(pcs + kG * kWarps);     // [kWarps] max ||v|| of valid tokens
  float *obuf = reinterpret_cast<float *>(smem);                 // [4][kG][kD], after the loop

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, t = lane & 3;
  const int t0 = s * a.chunk;
  const int64_t grp = (int64_t)b * a.hkv + h;
  const int64_t cap = min(a.k.capacity, a.v.capacity);
  constexpr unsigned FB = KP::regs * 32 * 4;  // the query fragments' bytes

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::br);
  int *fail = reinterpret_cast<int *>(smem + SM::br + 16);
  int *nlead_s = fail + 1;
  // Contiguous layout: the first sub-chunk's blocks are consecutive slots known before the
  // sequence length (bounded by the arrays only), so their copies start at once; blocks past the
  // sequence are masked later like any other.
  int early = 0;
  int64_t base0 = 0;
  if (!a.block_table) {
    base0 = ((int64_t)b * a.hkv + h) * a.ctx_stride + t0;
    int64_t nb = base0 < cap ? (cap - base0) / 16 : 0;
    const int lim = min(SM::NB, a.chunk / 16);
    early = (int)(nb < lim ? nb : lim);
  }
  if (tid == 0) {
    mbar_init(&bars[0], StageArrays<QJL>::n);
    mbar_init(&bars[1], StageArrays<QJL>::n);
    mbar_init(&bars[4], 1);  // the merge's copies (br + 32)
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    *fail = 0;
  }
  // Launched as a programmatic dependent of the query-fragment kernel: everything above overlaps
  // its tail; the caches (appended rows), fragments and counters are read only after this.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  __syncthreads();
  if (early > 0 && warp < StageArrays<QJL>::n && lane == 0) {
    const char *src;
    size_t doff;
    unsigned per;
    int64_t sstride;
    stage_array<BK, BV, QJL>(a, warp, src, doff, per, sstride);
    mbar_expect_arrive(&bars[0], per * (unsigned)early + (warp == 0 ? FB : 0u));
    bulk_g2s(smem + doff, src + base0 * sstride, per * (unsigned)early, &bars[0]);
    if (warp == 0) bulk_g2s(smem + SM::kf, kfrag + grp * KP::regs * 32, FB, &bars[0]);
  }
  int L = a.seq_lens[b];
  L = L < 0 ? 0 : (L > a.max_len ? a.max_len : L);
  const int t1 = min(L, t0 + a.chunk);
  const int nsub = t1 > t0 ? (t1 - t0 + kSub - 1) / kSub : 0;
  // the CTA's blocks: first slot, or -1 past the sequence or the arrays
  const int nblk = (t1 - t0 + 15) / 16;
  if (tid < SM::MAXBLK) {
    int64_t base = -1;
    if (tid < nblk) {
      base = token_slot(a, b, h, t0 + 16 * tid);
      if (base < 0 || base + 16 > cap) base = -1;
    }
    vball[tid] = base;
    // contiguous layout: the leading run of valid blocks (consecutive slots)
    const unsigned inval = __ballot_sync(TQ_FULL_MASK, base < 0);
    if ((tid & 31) == 0) nlead_s[tid >> 5] = inval ? __ffs(inval) - 1 : 32;
  }
  if (tid < kG) {
    hM[tid] = -INFINITY;
    hL[tid] = 0.f;
  }
  __syncthreads();
  const int nlead = nlead_s[0] < 32 ? nlead_s[0] : 32 + nlead_s[1];
  if (early == 0 && warp < StageArrays<QJL>::n && nsub > 0) {
    // the first sub-chunk (paged layout), and the query fragments (one copy per CTA) on the same
    // barrier
    stage_sub<BK, BV, QJL>(a, 0, vball, nlead, smem, &bars[0], FB);
    if (warp == 0 && lane == 0) bulk_g2s(smem + SM::kf, kfrag + grp * KP::regs * 32, FB, &bars[0]);
  }
  if (early > 0 && nsub == 0) {
    // an empty range still owns the early copies in flight: they land before the buffers are
    // reused for the partials
    if (!__syncthreads_and(mbar_wait_bounded(&bars[0], 0u))) {
      if (tid == 0) {
        atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
        mbar_wait_bounded(&bars[0], 0u);
      }
      __syncthreads();
    }
  }
  // Test hook (tq_debug_wait_probe): one bounded wait on the merge barrier, armed for bytes that
  // no copy sends, so that it runs out while the first sub-chunk's copies are in flight; the CTA
  // then takes the same abort path as a staging timeout (flag, drain its copies, return).
  const int probe = g_tq_wait_probe;
  if (probe > 0) {
    if (tid == 0) {
      mbar_expect_arrive(&bars[4], 16u);
      bool ok = false;
      for (int i = 0; i < probe && !ok; ++i) ok = mbar_try_wait(&bars[4], 0u);
      if (!ok) *fail = 1;
    }
    __syncthreads();
    if (*fail) {
      if (tid == 0) {
        atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
        if (nsub > 0 || early > 0) mbar_wait_bounded(&bars[0], 0u);
      }
      __syncthreads();
      return;
    }
  }
  // the query constants (2^-F_code, 2^-F_sign, Cq, Cp per head), read from shared memory where
  // used (published by the first sub-chunk's barrier)
  float *kcs = hL + kG;  // [16]
  if (tid < 16) kcs[tid] = kconst[grp * 16 + tid];

  // value accumulators of this thread: head t, coordinates jb + 2 mt + r
  const int ch = warp & 1, bgrp = warp >> 1;
  const int jb = 64 * ch + 8 * gid;
  float o[4][2];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) o[mt][0] = o[mt][1] = 0.f;

  for (int sc = 0; sc < nsub; ++sc) {
    const int cur = sc & 1;
    const int tk0 = t0 + sc * kSub;
    if (warp < StageArrays<QJL>::n && sc + 1 < nsub)
      stage_sub<BK, BV, QJL>(a, sc + 1, vball, nlead, smem + (cur ^ 1) * SM::buf, &bars[cur ^ 1], 0u);
    if (!mbar_wait_bounded(&bars[cur], (unsigned)(sc >> 1) & 1u)) *fail = 1;
    __syncthreads();
    if (*fail) {
      // the copies did not land in time: report, give the ones in flight a bounded time to
      // finish (they write this CTA's shared memory), and leave without writing partials
      if (tid == 0) {
        atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
        mbar_wait_bounded(&bars[cur], (unsigned)(sc >> 1) & 1u);
        if (sc + 1 < nsub) mbar_wait_bounded(&bars[cur ^ 1], (unsigned)((sc + 1) >> 1) & 1u);
      }
      __syncthreads();
      return;
    }
    const unsigned char *sb = smem + cur * SM::buf;
    const uint32_t *skc = reinterpret_cast<const uint32_t *>(sb + SM::kc);
    const uint32_t *sks = reinterpret_cast<const uint32_t *>(sb + SM::ks);
    const float *skn = reinterpret_cast<const float *>(sb + SM::kn);
    const float *skr = reinterpret_cast<const float *>(sb + SM::kr);
    const uint32_t *svc = reinterpret_cast<const uint32_t *>(sb + SM::vc);
    const float *svn = reinterpret_cast<const float *>(sb + SM::vn);
    const int64_t *vb = vball + NB * sc;  // validity of this sub-chunk's blocks

    // ------------------------------------------------------------ phase 1: logits (keys x heads)
    {
      // warp w: blocks 2w and 2w + 1; the query fragments of one (plane, k-step) serve both.
      // A = the key words masked in place (bytes 0 or 2^shift; B carries 2^-shift).
      int acc[2][2][2][4];  // [block][plane type][n-tile][c]
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
          for (int y = 0; y < 2; ++y)
#pragma unroll
            for (int z = 0; z < 4; ++z) acc[kb][x][y][z] = 0;
      uint32_t w[2][2][KP::all];
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int i = (2 * warp + kb) * 16 + gid + 8 * r;
#pragma unroll
          for (int P = 0; P < BK; ++P) w[kb][r][P] = skc[i * SM::KCW + P * 4 + t];
          if constexpr (BK == 3) w[kb][r][3] = w[kb][r][0] ^ w[kb][r][1] ^ w[kb][r][2];
          if constexpr (QJL) w[kb][r][KP::code] = sks[i * SM::KSW + t];
        }
#pragma unroll
      for (int P = 0; P < KP::all; ++P) {
        const int pt = (QJL && P == KP::code) ? 1 : 0;
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          const uint4 f = kf4[(P * 4 + st) * 32 + lane];
          const uint32_t mlo = 0x01010101u << st, mhi = 0x01010101u << (st + 4);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
            const uint32_t a0 = w[kb][0][P] & mlo, a1 = w[kb][1][P] & mlo;
            const uint32_t a2 = w[kb][0][P] & mhi, a3 = w[kb][1][P] & mhi;
            mma_u8s8(acc[kb][pt][0], a0, a1, a2, a3, f.x, f.y);
            mma_u8s8(acc[kb][pt][1], a0, a1, a2, a3, f.z, f.w);
          }
        }
      }
      float lmax = -INFINITY, nvmax = 0.f;
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        const int blk = 2 * warp + kb;
        const bool bok = vb[blk] >= 0;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int i = blk * 16 + gid + 8 * r;
          const float dc = (float)acc[kb][0][0][2 * r] + 256.f * (float)acc[kb][0][0][2 * r + 1] +
                           65536.f * (float)acc[kb][0][1][2 * r] + 16777216.f * (float)acc[kb][0][1][2 * r + 1];
          float sc2 = fmaf(dc, kcs[t], -kcs[8 + t]);
          if constexpr (QJL) {
            const float ds = (float)acc[kb][1][0][2 * r] + 256.f * (float)acc[kb][1][0][2 * r + 1] +
                             65536.f * (float)acc[kb][1][1][2 * r] + 16777216.f * (float)acc[kb][1][1][2 * r + 1];
            sc2 = fmaf(kc.qjl_scale * skr[i], fmaf(ds, kcs[4 + t], -kcs[12 + t]), sc2);
          }
          const bool ok = bok && tk0 + i < t1;
          const float lgt = ok ? a.scale * skn[i] * sc2 : -INFINITY;
          lg[t * kLgS + i] = lgt;
          lmax = fmaxf(lmax, lgt);
          if (ok) nvmax = fmaxf(nvmax, svn[i]);
        }
      }
      // this warp's largest logit per head (lanes sharing t hold the same head)
#pragma unroll
      for (int m = 4; m <= 16; m <<= 1) {
        lmax = fmaxf(lmax, __shfl_xor_sync(TQ_FULL_MASK, lmax, m));
        nvmax = fmaxf(nvmax, __shfl_xor_sync(TQ_FULL_MASK, nvmax, m));
      }
      if (gid == 0) pmax[t * kWarps + warp] = lmax;
      if (lane == 0) pnv[warp] = nvmax;
    }
    __syncthreads();

    // ------------------------------------------------------------ phase 2: weights, value fragments
    // Each warp weights its own two blocks (tokens 32 w ..) and builds their value-MMA B
    // fragments; the fixed-point scale comes from the sub-chunk's largest ||v|| (W <= ||v||
    // since w <= 1), so no cross-warp step is needed in between.
    {
      const int g = lane & 3;  // lane = (head lane & 3, tokens lane / 4 + 8 k)
      const float Mnew = fmaxf(hM[g], max8(pmax + g * kWarps));
      float sw = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = 32 * warp + (lane >> 2) + 8 * k;
        const float l = lg[g * kLgS + i];
        const float wgt = l == -INFINITY ? 0.f : __expf(l - Mnew);
        lg[g * kLgS + i] = l == -INFINITY ? 0.f : wgt * svn[i];  // masked slots may hold stale bytes
        sw += wgt;
      }
#pragma unroll
      for (int m = 4; m <= 16; m <<= 1) sw += __shfl_xor_sync(TQ_FULL_MASK, sw, m);
      if (lane < kG) psw[g * kWarps + warp] = sw;
      if constexpr (BV == 3) {
        // (plane 2, parity) words of this warp's two blocks, parity = p0 ^ p1 ^ p2
#pragma unroll
        for (int k = 0; k < 2 * kD / 32; ++k) {
          const int idx = lane + 32 * k;
          const int kb = 2 * warp + (idx >> 7), j = idx & (kD - 1);
          const uint32_t A = svc[kb * SM::VBW + j];
          const uint32_t hw = svc[kb * SM::VBW + kD + (j >> 1)] >> (16 * (j & 1));
          const uint32_t par = A ^ (A >> 16) ^ hw;
          sx1[kb * SM::X1W + j] = __byte_perm(hw, par, 0x5410);
        }
      }
      __syncwarp();
      // B fragments of the value MMAs.  Lane (gid, t): column = (head gid/2, limb gid&1).  The
      // k index runs over (token, plane) pairs in the order the value words give them:
      // register 0 = tokens t, t+8 of the low plane, then of the high plane; register 1 = the
      // same for tokens t+4, t+12.  Byte = limb of X = floor(W 2 e_P sc + dither), dithered so
      // that the many sub-unit tail weights are unbiased rather than all rounded down.
      const int gh = gid >> 1, l = gid & 1;
      float sc, inv;
      weight_scale(max8(pnv) * 2.f * vc.plane_coef_max, sc, inv);
      float C[2 * VT];
#pragma unroll
      for (int P = 0; P < 2 * VT; ++P) C[P] = 2.f * sc * vc.plane_coef[P];
      const uint32_t sel = (uint32_t)l | ((uint32_t)(4 + l) << 4);  // byte l of two words
      const uint32_t key0 = ((uint32_t)grp * (uint32_t)a.max_len + (uint32_t)tk0) * 4u + (uint32_t)gh;
      uint32_t xs = 0;  // sum of this lane's X values
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kb = 2 * warp + kk;
        const float *wr = &lg[gh * kLgS + kb * 16];
        const int toks[4] = {t, t + 8, t + 4, t + 12};
        float W[4], dz[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          W[i] = wr[toks[i]];
          dz[i] = dither(key0 + 4u * (uint32_t)(kb * 16 + toks[i]));
        }
        uint32_t reg[2 * VT];
#pragma unroll
        for (int x = 0; x < VT; ++x)
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int i0 = 2 * rr, i1 = 2 * rr + 1;  // the two tokens of this register
            const uint32_t x0 = floor_bits(fmaf(W[i0], C[2 * x], dz[i0]));
            const uint32_t x1 = floor_bits(fmaf(W[i1], C[2 * x], dz[i1]));
            const uint32_t x2 = floor_bits(fmaf(W[i0], C[2 * x + 1], dz[i0]));
            const uint32_t x3 = floor_bits(fmaf(W[i1], C[2 * x + 1], dz[i1]));
            reg[2 * x + rr] = __byte_perm(__byte_perm(x0, x1, sel), __byte_perm(x2, x3, sel), 0x5410);
            xs += (x0 + x1) + (x2 + x3) - 4u * 0x4B000000u;  // the integers themselves
          }
        vfrag[kb * 32 + lane] = VT == 2 ? make_uint4(reg[0], reg[1], reg[2 * VT - 2], reg[2 * VT - 1])
                                        : make_uint4(reg[0], reg[1], 0u, 0u);
      }
      // the codebook's constant term uses the same integers: sum X per head (limb-0 lanes)
      uint32_t mine = l == 0 ? xs : 0u;
      mine += __shfl_xor_sync(TQ_FULL_MASK, mine, 1);
      mine += __shfl_xor_sync(TQ_FULL_MASK, mine, 2);
      mine += __shfl_xor_sync(TQ_FULL_MASK, mine, 4);
      if (t == 0 && l == 0) pcs[gh * kWarps + warp] = (int)mine;
    }
    __syncthreads();

    // ------------------------------------------------------------ phase 3: value sum
    // warp w: coordinate half ch = w & 1 (64 coordinates = 4 m-tiles) and blocks bgrp + 4 k.
    // In m-tile mt, row gid <-> coordinate 64 ch + 8 gid + 2 mt and row gid + 8 <-> the next one.
    {
      const uint32_t mlo = 1u << (7 - t), mhi = 1u << (3 - t);
      int accv[4][VT][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int x = 0; x < VT; ++x)
#pragma unroll
          for (int z = 0; z < 4; ++z) accv[mt][x][z] = 0;
#pragma unroll
      for (int kk = 0; kk < NB / 4; ++kk) {
        const int kb = bgrp + 4 * kk;
        if (vb[kb] < 0) continue;
        uint32_t X[VT][8];
        {
          const uint4 u0 = *reinterpret_cast<const uint4 *>(svc + kb * SM::VBW + jb);
          const uint4 u1 = *reinterpret_cast<const uint4 *>(svc + kb * SM::VBW + jb + 4);
          X[0][0] = u0.x; X[0][1] = u0.y; X[0][2] = u0.z; X[0][3] = u0.w;
          X[0][4] = u1.x; X[0][5] = u1.y; X[0][6] = u1.z; X[0][7] = u1.w;
        }
        if constexpr (BV == 3) {
          const uint4 u0 = *reinterpret_cast<const uint4 *>(sx1 + kb * SM::X1W + jb);
          const uint4 u1 = *reinterpret_cast<const uint4 *>(sx1 + kb * SM::X1W + jb + 4);
          X[VT - 1][0] = u0.x; X[VT - 1][1] = u0.y; X[VT - 1][2] = u0.z; X[VT - 1][3] = u0.w;
          X[VT - 1][4] = u1.x; X[VT - 1][5] = u1.y; X[VT - 1][6] = u1.z; X[VT - 1][7] = u1.w;
        }
        const uint4 fb = vfrag[kb * 32 + lane];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
          for (int x = 0; x < VT; ++x) {
            // token bits t, t+8 (and t+4, t+12) of both planes moved to bit 7 of each byte by a
            // multiply (the FMA pipe) and kept by one AND: bytes 0 or 128
            const uint32_t r0 = X[x][2 * mt], r1 = X[x][2 * mt + 1];
            const uint32_t a0 = mul_lo(r0, mlo) & 0x80808080u, a1 = mul_lo(r1, mlo) & 0x80808080u;
            const uint32_t a2 = mul_lo(r0, mhi) & 0x80808080u, a3 = mul_lo(r1, mhi) & 0x80808080u;
            mma_u8u8(accv[mt][x], a0, a1, a2, a3, x == 0 ? fb.x : fb.z, x == 0 ? fb.y : fb.w);
          }
      }
      // accv[mt][x][c]: c0/c1 = (coordinate jb + 2 mt, head t, limb 0/1), c2/c3 = (+1, ...):
      // 128 sum_tok X b over the word type's two planes.  With s = 2b - 1 the codebook's
      // constant term is -(1/2) sum X, added once per sub-chunk by the bgrp 0 warps.
      const float Mold = hM[t], Mnew = fmaxf(Mold, max8(pmax + t * kWarps));
      const float al = Mnew == -INFINITY ? 1.f : __expf(Mold - Mnew);
      float sct, inv;
      weight_scale(max8(pnv) * 2.f * vc.plane_coef_max, sct, inv);
      int cs = 0;
#pragma unroll
      for (int w2 = 0; w2 < kWarps; ++w2) cs += pcs[t * kWarps + w2];
      const float cterm = bgrp == 0 ? 64.f * (float)cs : 0.f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float v = 0.f;
#pragma unroll
          for (int x = 0; x < VT; ++x) v += (float)accv[mt][x][2 * r] + 256.f * (float)accv[mt][x][2 * r + 1];
          o[mt][r] = fmaf(o[mt][r], al, (v - cterm) * inv);
        }
    }
    __syncthreads();  // the buffers, lg, vfrag and the per-warp partials are reused next
    if (warp == kWarps - 1 && lane < kG) {
      // head `lane`'s running maximum and sum, from this sub-chunk's per-warp partials (read
      // before the next sub-chunk's phase 1 rewrites them, published by its first barrier);
      // the last warp does it, as it issues no copies
      const float Mold = hM[lane], Mnew = fmaxf(Mold, max8(pmax + lane * kWarps));
      const float al = Mnew == -INFINITY ? 1.f : __expf(Mold - Mnew);
      float swh = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kWarps; ++w2) swh += psw[lane * kWarps + w2];
      hM[lane] = Mnew;
      hL[lane] = hL[lane] * al + swh;
    }
  }

  // ---------------------------------------------------------------- partials of the 4 heads
  __syncthreads();
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int r = 0; r < 2; ++r) obuf[(bgrp * kG + t) * kD + jb + 2 * mt + r] = o[mt][r];
  __syncthreads();
  for (int i = tid; i < kG * kD; i += kThreads) {
    const int g = i / kD, j = i % kD;
    const float v = obuf[(0 * kG + g) * kD + j] + obuf[(1 * kG + g) * kD + j] + obuf[(2 * kG + g) * kD + j] +
                    obuf[(3 * kG + g) * kD + j];
    const int64_t pb = (((int64_t)b * a.hq + (int64_t)h * kG + g) * a.splits + s) * (kD + 4);
    part[pb + 2 + j] = v;
  }
  if (tid < kG) {
    const int64_t pb = (((int64_t)b * a.hq + (int64_t)h * kG + tid) * a.splits + s) * (kD + 4);
    part[pb] = hM[tid];
    part[pb + 1] = hL[tid];
  }
  if (a.out == nullptr) return;

  // ---------------------------------------------------------------- merge (last CTA of the group)
  // The last CTA of this (sequence, KV head) to finish merges the splits of its 4 heads with
  // their log-sum-exp weights and undoes the rotation once:
  //   o = D_V (1/sqrt d) H (sum_s e^{m_s - M} o~_s) / (sum_s e^{m_s - M} l_s).
  // release: the barrier orders every thread's partial stores before thread 0's fence, which
  // (cumulatively) orders them before the count at device scope
  __syncthreads();
  int *last = nlead_s + 2;
  if (tid == 0) {
    __threadfence();
    *last = atomicAdd(&a.counter[grp], 1) == a.splits - 1;
    if (*last) {
      __threadfence();  // acquire: the other CTAs' partials are read after this ...
      asm volatile("fence.proxy.async.global;\n" ::: "memory");  // ... by the bulk copies too
    }
  }
  __syncthreads();
  if (!*last) return;
  // The group's partial rows (kD + 4 floats: m, l, o~, pad) pass through shared memory in
  // batches of up to `nb` splits (one bulk copy per head and batch).  While a batch's copies are
  // in flight, warp g < 4 reads head g's (m, l) straight from L2 and forms the merge factors
  // e^{m_s - M}; then warps g and g + 4 accumulate head g's even and odd splits (lane holding
  // coordinates lane + 32 k), and warp g adds warp g + 4's share.
  constexpr int PR = kD + 4;
  float *stg = reinterpret_cast<float *>(smem);  // [kG][nb][PR], then fs [kG][nb]
  const int nb = (int)(SM::vb / ((size_t)kG * (PR + 1) * 4));
  float *fs = stg + (size_t)kG * nb * PR;
  float *rfac = hM;  // [kG] rescale of the running sums for the batch
  const int64_t pg = ((int64_t)b * a.hq + (int64_t)h * kG) * a.splits * PR;
  const int hg = warp & (kG - 1), par = warp >> 2;
  float sgn[4];  // the rotation signs of this lane's output coordinates, loaded early
#pragma unroll
  for (int k = 0; k < 4; ++k) sgn[k] = vc.signs[lane + 32 * k] * vc.inv_sqrt_d;
  float M = -INFINITY, Lsum = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s0 = 0; s0 < a.splits; s0 += nb) {
    const int n = min(nb, a.splits - s0);
    // each head's n rows are contiguous in the partials: one bulk copy per head
    if (tid == 0) mbar_expect_arrive(&bars[4], (unsigned)(kG * n * PR * 4));
    __syncthreads();
    if (tid < kG)
      bulk_g2s(stg + (size_t)tid * n * PR, part + pg + ((int64_t)tid * a.splits + s0) * PR, (unsigned)(n * PR * 4),
               &bars[4]);
    if (warp < kG) {
      const float *pb = part + pg + ((int64_t)warp * a.splits + s0) * PR;
      float Mb = M, Lb = 0.f;
      if (n <= 64) {
        // one round trip: up to two (m, l) pairs per lane held in registers
        float m2[2], l2[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int sp = lane + 32 * j;
          m2[j] = sp < n ? __ldcg(pb + (int64_t)sp * PR) : -INFINITY;
          l2[j] = sp < n ? __ldcg(pb + (int64_t)sp * PR + 1) : 0.f;
          Mb = fmaxf(Mb, m2[j]);
        }
        Mb = warp_max_f(Mb);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int sp = lane + 32 * j;
          const float f = m2[j] == -INFINITY ? 0.f : __expf(m2[j] - Mb);
          if (sp < n) fs[warp * nb + sp] = f;
          Lb = fmaf(f, l2[j], Lb);
        }
      } else {
        for (int sp = lane; sp < n; sp += 32) Mb = fmaxf(Mb, __ldcg(pb + (int64_t)sp * PR));
        Mb = warp_max_f(Mb);
        for (int sp = lane; sp < n; sp += 32) {
          const float ms = __ldcg(pb + (int64_t)sp * PR);
          const float f = ms == -INFINITY ? 0.f : __expf(ms - Mb);
          fs[warp * nb + sp] = f;
          Lb = fmaf(f, __ldcg(pb + (int64_t)sp * PR + 1), Lb);
        }
      }
      Lb = warp_sum_f(Lb);
      const float r = Mb == -INFINITY ? 1.f : __expf(M - Mb);  // 0 while M is -inf
      Lsum = fmaf(Lsum, r, Lb);
      M = Mb;
      if (lane == 0) rfac[warp] = r;
    }
    if (!__syncthreads_and(mbar_wait_bounded(&bars[4], (unsigned)(s0 / nb) & 1u))) {
      if (tid == 0) {
        atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
        mbar_wait_bounded(&bars[4], (unsigned)(s0 / nb) & 1u);
      }
      __syncthreads();
      return;
    }
    {
      const float r = rfac[hg];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] *= r;
      const float *rows = stg + (size_t)hg * n * PR;
      const float *fg = fs + hg * nb;
#pragma unroll 2
      for (int sp = par; sp < n; sp += 2) {
        const float f = fg[sp];
        const float *row = rows + sp * PR + 2 + lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = fmaf(f, row[32 * k], acc[k]);
      }
    }
    __syncthreads();  // the batch buffer is refilled next (or the exchange area is used)
  }
  // warp g + 4 hands its share of acc to warp g through shared memory (same scale M)
  float *xw = stg + (size_t)hg * (4 * 32);
  if (par == 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) xw[32 * k + lane] = acc[k];
  }
  __syncthreads();
  if (warp >= kG) return;
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] += xw[32 * k + lane];
  // o = D_V (1/sqrt d) H (acc / L): butterflies of span 32 and 64 within the lane, 1..16 across
  // lanes (value k of lane i is coordinate i + 32 k)
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] *= inv;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float o = __shfl_xor_sync(TQ_FULL_MASK, acc[k], m);
      acc[k] = upper ? o - acc[k] : acc[k] + o;
    }
  }
  {
    const float u0 = acc[0] + acc[1], u1 = acc[0] - acc[1], u2 = acc[2] + acc[3], u3 = acc[2] - acc[3];
    acc[0] = u0 + u2;
    acc[1] = u1 + u3;
    acc[2] = u0 - u2;
    acc[3] = u1 - u3;
  }
  float *dst = a.out + ((int64_t)b * a.hq + (int64_t)h * kG + warp) * kD;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = lane + 32 * k;
    dst[j] = sgn[k] * acc[k];
  }
}

template <int BK, int BV, bool QJL>
cudaError_t launch_mma(const TqConsts &kc, const TqConsts &vc, const MmaArgs &a, dim3 grid,
                       const uint32_t *kfrag, const float *kconst, float *part, cudaStream_t st) {
  const size_t smem = MmaSmem<BK, BV, QJL>::total;
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(attend_mma_kernel<BK, BV, QJL>),
                                       (int)smem);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: the grid may start while the preceding kernel on the stream
  // (the query-fragment or decode-prep kernel) finishes; the kernel waits for it before use.  With
  // per-kernel profiling on, an event sits between the two kernels and a plain launch is used.
  if (tq_prof_on()) {
    attend_mma_kernel<BK, BV, QJL><<<grid, kThreads, smem, st>>>(kc, vc, a, kfrag, kconst, part);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attend_mma_kernel<BK, BV, QJL>, kc, vc, a, kfrag, kconst, part);
}

template <int BK, int BV, bool QJL>
cudaError_t launch_fast(const TqConsts &kc, const TqConsts &vc, const MmaArgs &a, int batch, const void *q,
                        int dtype, uint32_t *kfrag, float *kconst, float *part, cudaStream_t st) {
  const unsigned groups = (unsigned)(batch * a.hkv);
  const size_t fsm = QJL ? sizeof(float) * kD * (kD + 4) : 0;
  if (fsm) {
    cudaError_t e0 = tq_smem_limit(reinterpret_cast<const void *>(kfrag_kernel<BK, QJL>), (int)fsm);
    if (e0 != cudaSuccess) return e0;
  }
  tq_prof_begin(TQK_ATTEND_FRAG, st);
  kfrag_kernel<BK, QJL><<<groups, kThreads, fsm, st>>>(kc, q, dtype, kfrag, kconst, a.counter);
  tq_prof_end(TQK_ATTEND_FRAG, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)a.splits, (unsigned)a.hkv, (unsigned)batch);
  tq_prof_begin(TQK_ATTEND_SPLIT, st);
  e = launch_mma<BK, BV, QJL>(kc, vc, a, grid, kfrag, kconst, part, st);
  tq_prof_end(TQK_ATTEND_SPLIT, st);
  return e;
}

}  // namespace

bool attn_fast_eligible(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc) {
  if (desc.n_kv_heads <= 0 || desc.n_q_heads != kG * desc.n_kv_heads) return false;
  if (kc.d != kD || vc.d != kD) return false;
  if (kc.layout != TQ_LAYOUT_ROWS || vc.layout != TQ_LAYOUT_BLOCK16) return false;
  if (kc.bits < 1 || kc.bits > 3 || (vc.bits != 2 && vc.bits != 3)) return false;
  if (kc.m != 0 && kc.m != kD) return false;
  if (!kc.fast_ok || !vc.fast_ok) return false;
  // the value weights are unsigned fixed point: every plane coefficient must be >= 0
  for (int P = 0; P < (vc.bits == 3 ? 4 : vc.bits); ++P)
    if (!(vc.plane_coef[P] >= 0.f)) return false;
  if (desc.block_table ? (desc.block_size % 16) != 0 : (desc.ctx_stride % 16) != 0) return false;
  return true;
}

int attn_fast_chunk(const tq_attn_desc &desc) {
  // Tokens per CTA (a multiple of 16): the 16-token blocks of all (sequence, KV head) rows split
  // evenly over two resident CTAs per SM, so that a uniform batch runs as one full wave; at least
  // 128 tokens (the fixed per-CTA work) and at most 1024 (long or ragged batches then run as
  // many short waves that the block scheduler balances).
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) sms = n;
  }
  const int64_t rows = (int64_t)desc.batch * desc.n_kv_heads;
  const int maxlen = desc.max_seq_len > 0 ? desc.max_seq_len : 1;
  const int64_t blocks = rows * ((maxlen + 15) / 16);
  const int64_t slots = 2 * (int64_t)sms;
  int64_t per = (blocks + slots - 1) / slots;
  per = per < 8 ? 8 : (per > 64 ? 64 : per);
  return (int)(16 * per);
}

size_t attn_fast_extra_bytes(const TqConsts &kc, const tq_attn_desc &desc) {
  const int planes = (kc.bits + (kc.bits == 3 ? 1 : 0)) + (kc.m > 0 ? 1 : 0);
  const int64_t groups = (int64_t)desc.batch * desc.n_kv_heads;
  return (size_t)tq_align_up(groups * planes * 16 * 32 * 4, 256) + (size_t)tq_align_up(groups * 16 * 4, 256) +
         (size_t)tq_align_up(groups * 4, 256);
}

cudaError_t launch_attend_fast(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc,
                               const AttnPlan &plan, const void *q, int dtype, void *extra,
                               float *partials, float *out, cudaStream_t st) {
  MmaArgs a;
  a.hq = desc.n_q_heads;
  a.hkv = desc.n_kv_heads;
  a.max_len = desc.max_seq_len;
  a.chunk = plan.chunk;
  a.splits = plan.splits;
  a.block_size = desc.block_size;
  a.max_blocks = desc.max_blocks;
  a.ctx_stride = desc.ctx_stride;
  a.scale = desc.scale != 0.f ? desc.scale : kc.inv_sqrt_d;
  a.seq_lens = desc.seq_lens;
  a.block_table = desc.block_table;
  a.k = desc.k;
  a.v = desc.v;
  const int planes = (kc.bits + (kc.bits == 3 ? 1 : 0)) + (kc.m > 0 ? 1 : 0);
  const int64_t groups = (int64_t)desc.batch * desc.n_kv_heads;
  uint32_t *kfrag = static_cast<uint32_t *>(extra);
  float *kconst = reinterpret_cast<float *>(static_cast<char *>(extra) +
                                            tq_align_up(groups * planes * 16 * 32 * 4, 256));
  a.counter = reinterpret_cast<int *>(reinterpret_cast<char *>(kconst) + tq_align_up(groups * 16 * 4, 256));
  a.out = out;
  const bool qjl = kc.m > 0;
#define TQ_FAST(BKV, BVV, Q)                                                                           \
  if (kc.bits == BKV && vc.bits == BVV && qjl == Q)                                                    \
    return launch_fast<BKV, BVV, Q>(kc, vc, a, desc.batch, q, dtype, kfrag, kconst, partials, st);
  TQ_FAST(1, 2, true) TQ_FAST(2, 2, true) TQ_FAST(3, 2, true)
  TQ_FAST(1, 3, true) TQ_FAST(2, 3, true) TQ_FAST(3, 3, true)
  TQ_FAST(1, 2, false) TQ_FAST(2, 2, false) TQ_FAST(3, 2, false)
  TQ_FAST(1, 3, false) TQ_FAST(2, 3, false) TQ_FAST(3, 3, false)
#undef TQ_FAST
  return cudaErrorInvalidValue;
}

namespace {
template <int BK, int BV, bool QJL>
cudaError_t launch_step(const TqConsts &kc, const TqConsts &vc, const MmaArgs &a, int batch, const void *knew,
                        const void *vnew, int kvdtype, int64_t nnew, const int64_t *slots, const void *q, int qdtype,
                        uint32_t *kfrag, float *kconst, float *part, cudaStream_t st) {
  const int nvb = (int)((nnew + (kThreads / 32) - 1) / (kThreads / 32));  // one value row per warp
  const int nkb = QJL ? (int)nnew : nvb;                                       // keys: see decode_prep_kernel
  const unsigned grid0 = (unsigned)(nkb + nvb + batch * a.hq);
  const size_t fsm = QJL ? sizeof(float) * kD * (kD + 4) : 0;
  if (fsm) {
    cudaError_t e0 = tq_smem_limit(reinterpret_cast<const void *>(decode_prep_kernel<BK, QJL>),
                                          (int)fsm);
    if (e0 != cudaSuccess) return e0;
  }
  tq_prof_begin(TQK_DECODE_PREP, st);
  decode_prep_kernel<BK, QJL><<<grid0, kThreads, fsm, st>>>(kc, vc, knew, vnew, kvdtype, nnew, slots, a.k, a.v, q,
                                                            qdtype, kfrag, kconst, a.counter, nkb, nvb);
  tq_prof_end(TQK_DECODE_PREP, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)a.splits, (unsigned)a.hkv, (unsigned)batch);
  tq_prof_begin(TQK_ATTEND_SPLIT, st);
  e = launch_mma<BK, BV, QJL>(kc, vc, a, grid, kfrag, kconst, part, st);
  tq_prof_end(TQK_ATTEND_SPLIT, st);
  return e;
}
}  // namespace

cudaError_t launch_decode_step_fast(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc,
                                    const AttnPlan &plan, const void *knew, const void *vnew, int kvdtype,
                                    int64_t nnew, const int64_t *slots, const void *q, int qdtype, void *extra,
                                    float *partials, float *out, cudaStream_t st) {
  MmaArgs a;
  a.hq = desc.n_q_heads;
  a.hkv = desc.n_kv_heads;
  a.max_len = desc.max_seq_len;
  a.chunk = plan.chunk;
  a.splits = plan.splits;
  a.block_size = desc.block_size;
  a.max_blocks = desc.max_blocks;
  a.ctx_stride = desc.ctx_stride;
  a.scale = desc.scale != 0.f ? desc.scale : kc.inv_sqrt_d;
  a.seq_lens = desc.seq_lens;
  a.block_table = desc.block_table;
  a.k = desc.k;
  a.v = desc.v;
  const int planes = (kc.bits + (kc.bits == 3 ? 1 : 0)) + (kc.m > 0 ? 1 : 0);
  const int64_t groups = (int64_t)desc.batch * desc.n_kv_heads;
  uint32_t *kfrag = static_cast<uint32_t *>(extra);
  float *kconst = reinterpret_cast<float *>(static_cast<char *>(extra) +
                                            tq_align_up(groups * planes * 16 * 32 * 4, 256));
  a.counter = reinterpret_cast<int *>(reinterpret_cast<char *>(kconst) + tq_align_up(groups * 16 * 4, 256));
  a.out = out;
  const bool qjl = kc.m > 0;
#define TQ_STEP(BKV, BVV, Q)                                                                                   \
  if (kc.bits == BKV && vc.bits == BVV && qjl == Q)                                                            \
    return launch_step<BKV, BVV, Q>(kc, vc, a, desc.batch, knew, vnew, kvdtype, nnew, slots, q, qdtype, kfrag, \
                                    kconst, partials, st);
  TQ_STEP(1, 2, true) TQ_STEP(2, 2, true) TQ_STEP(3, 2, true)
  TQ_STEP(1, 3, true) TQ_STEP(2, 3, true) TQ_STEP(3, 3, true)
  TQ_STEP(1, 2, false) TQ_STEP(2, 2, false) TQ_STEP(3, 2, false)
  TQ_STEP(1, 3, false) TQ_STEP(2, 3, false) TQ_STEP(3, 3, false)
#undef TQ_STEP
  return cudaErrorInvalidValue;
}

extern "C" tq_status tq_device_status(int32_t device, int32_t *flags, int32_t clear) {
  if (!flags) return tq_fail(TQ_EINVAL, "flags is NULL");
  DeviceScope dev_scope;
  tq_status st = dev_scope.enter(device);
  if (st != TQ_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  int v = 0, vr = 0, vm = 0, vt = 0;
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_tq_device_flags, sizeof(int));
  if (e == cudaSuccess) e = rotate_device_flags(&vr, clear != 0);
  if (e == cudaSuccess) e = search_mma_device_flags(&vm, clear != 0);
  if (e == cudaSuccess) e = search_tc_device_flags(&vt, clear != 0);
  if (e == cudaSuccess && clear) {
    const int z = 0;
    e = cudaMemcpyToSymbol(g_tq_device_flags, &z, sizeof(int));
  }
  v |= vr | vm | vt;
  if (e != cudaSuccess) return tq_fail(TQ_ECUDA, "device status: %s", cudaGetErrorString(e));
  *flags = v;
  if (v & TQ_DEVFLAG_STAGING_TIMEOUT)
    return tq_fail(TQ_ETIMEOUT, "a kernel on device %d gave up waiting for its asynchronous copies and left "
                                "its outputs unwritten%s", device, clear ? " (flag now cleared)" : "");
  return TQ_OK;
}

extern "C" tq_status tq_debug_wait_probe(int32_t device, int32_t polls) {
  if (polls < 0) return tq_fail(TQ_EINVAL, "polls < 0");
  DeviceScope dev_scope;
  tq_status st = dev_scope.enter(device);
  if (st != TQ_OK) return st;
  return tq_cuda_check(cudaMemcpyToSymbol(g_tq_wait_probe, &polls, sizeof(int)), "wait probe");
}
