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

struct MmaArgs {
  int hq, hkv, max_len, chunk, splits, block_size, max_blocks;
  int64_t ctx_stride;
  float scale;
  const int32_t *seq_lens;
  const int32_t *block_table;
  tq_packed k, v;
  int *counter;  // per (sequence, KV head): CTAs done (zeroed by the query-fragment kernel)
  float *out;    // final output when the kernel merges its splits itself, else null
  float sparse_v;  // Sparse V threshold on the softmax weights (0 = off)
  int kn4, vn4;    // log2 of the bytes of one stored K / V norm: 2 (fp32) or 1 (fp16)
};

// Norm i of a staged array (fp16 when NH, else fp32).
template <bool NH>
__device__ __forceinline__ float staged_norm(const unsigned char *base, int i) {
  if constexpr (NH)
    return __half2float(reinterpret_cast<const __half *>(base)[i]);
  else
    return reinterpret_cast<const float *>(base)[i];
}

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

// 1 + u, u uniform in [0, 1), from a 32-bit key: u = the fractional part of key * (golden ratio)
// to 23 bits (5184445 / 2^23), a low-discrepancy sequence over consecutive keys (deterministic
// dither for rounding), as the mantissa of a float in [1, 2): one multiply and one logic op.
__device__ __forceinline__ float dither1(uint32_t x) { return __uint_as_float(0x3F800000u | ((x * 5184445u) & 0x7FFFFFu)); }


// A float's order-preserving int (for an integer atomicMax over floats, -inf included) and back.
__device__ __forceinline__ int ord_float(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float unord_float(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF); }

// Two fp32 FMAs in one packed instruction (f32x2): d_i = a_i b + c_i, each rounded as fmaf.
__device__ __forceinline__ void fma2(float a0, float a1, float b, float c0, float c1, float &d0, float &d1) {
  uint64_t r;
  asm("{\n .reg .b64 pa, pb, pc;\n mov.b64 pa, {%1, %2};\n mov.b64 pb, {%3, %3};\n mov.b64 pc, {%4, %5};\n"
      " fma.rn.f32x2 %0, pa, pb, pc;\n}"
      : "=l"(r)
      : "r"(__float_as_uint(a0)), "r"(__float_as_uint(a1)), "r"(__float_as_uint(b)), "r"(__float_as_uint(c0)),
        "r"(__float_as_uint(c1)));
  d0 = __uint_as_float((uint32_t)r);
  d1 = __uint_as_float((uint32_t)(r >> 32));
}

// floor(w_i c + z_i - 1) for a pair, in two packed instructions, as the low mantissa bits of
// 2^23 + that integer (a round-down add on the FMA pipe instead of a float-to-integer conversion;
// the result's bytes 0 and 1 are the integer's): z_i = 1 + dither in [1, 2), so the sum plus
// 2^23 - 1 lies on the integer grid of [2^23, 2^24).
__device__ __forceinline__ void fma_floor2(float w0, float w1, float c, float z0, float z1, uint32_t &x0,
                                           uint32_t &x1) {
  uint64_t r;
  asm("{\n .reg .b64 pa, pb, pc, pm, pt;\n mov.b64 pa, {%1, %2};\n mov.b64 pb, {%3, %3};\n"
      " mov.b64 pc, {%4, %5};\n fma.rn.f32x2 pt, pa, pb, pc;\n mov.b64 pm, {%6, %6};\n"
      " add.rm.f32x2 %0, pt, pm;\n}"
      : "=l"(r)
      : "r"(__float_as_uint(w0)), "r"(__float_as_uint(w1)), "r"(__float_as_uint(c)), "r"(__float_as_uint(z0)),
        "r"(__float_as_uint(z1)), "r"(0x4AFFFFFEu));
  x0 = (uint32_t)r;
  x1 = (uint32_t)(r >> 32);
}

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
  // S (for p = S q') is copied asynchronously while q' is formed (sS null: read from global)
  if constexpr (QJL)
    if (sS) stage_rows_padded_async(sS, kc.S, kD, kD);
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
    if (sS) stage_async_wait();
    __syncthreads();
    const int i = tid & (kD - 1), gp = tid >> 7;
    float p0 = 0.f, p1 = 0.f;
    if (sS) {
      const float4 *Srow = reinterpret_cast<const float4 *>(sS + i * (kD + 4));
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
    } else {
      // S transposed in global memory: consecutive rows i per warp, coalesced (same order of sums)
#pragma unroll 32
      for (int j = 0; j < kD; ++j) {
        const float sv = kc.St[j * kc.m + i];
        p0 = fmaf(sv, qs[2 * gp][j], p0);
        p1 = fmaf(sv, qs[2 * gp + 1][j], p1);
      }
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
  if constexpr (QJL)
    if (sS) stage_rows_padded_async(sS, kc.S, kD, kD);
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
    if (sS) stage_async_wait();
    __syncthreads();
    if (tid < kD) {
      float p0 = 0.f;
      if (sS) {
        const float4 *Srow = reinterpret_cast<const float4 *>(sS + tid * (kD + 4));
#pragma unroll 8
        for (int j4 = 0; j4 < kD / 4; ++j4) {
          const float4 sv = Srow[j4];
          p0 = fmaf(sv.x, qs[4 * j4], p0);
          p0 = fmaf(sv.y, qs[4 * j4 + 1], p0);
          p0 = fmaf(sv.z, qs[4 * j4 + 2], p0);
          p0 = fmaf(sv.w, qs[4 * j4 + 3], p0);
        }
      } else {
#pragma unroll 32
        for (int j = 0; j < kD; ++j) p0 = fmaf(kc.St[j * kc.m + tid], qs[j], p0);
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
// blocks build the query fragments: one query head each (`per_head`, for small batches, so that
// more blocks share the latency) or one (sequence, KV head) group each.  The jobs are
// independent, so their latencies overlap instead of adding up.  Small launches stage S in each
// block's shared memory; large ones read its transposed copy from global memory (coalesced; it
// stays in L1 and L2), so that many blocks fit on an SM.
template <int BK, bool QJL>
__global__ void __launch_bounds__(kThreads)
decode_prep_kernel(TqConsts kc, TqConsts vc, const void *__restrict__ knew, const void *__restrict__ vnew,
                   int kvdtype, int64_t nnew, const int64_t *__restrict__ slots, tq_packed kp, tq_packed vp,
                   const void *__restrict__ q, int qdtype, uint32_t *__restrict__ kfrag,
                   float *__restrict__ kconst, int *__restrict__ counter, int nkb, int nvb, int per_head) {
  extern __shared__ __align__(16) float sS[];  // S staged per block for small launches (per_head)
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");  // the attention grid may start
  float *ss = per_head ? sS : nullptr;
  const int bid = blockIdx.x;
  if (bid < nkb) {
    // keys: with QJL one row per block (warps 0-3 share its projection), else 8 rows per block
    rotate_rows<kD>(kc, ROT_ENCODE, knew, kvdtype, nnew, kD, slots, kp.capacity, static_cast<uint32_t *>(kp.codes),
                    kp.norm, kp.rnorm, nullptr, QJL ? static_cast<uint32_t *>(kp.signs) : nullptr, bid, ss, QJL);
  } else if (bid < nkb + nvb) {
    rotate_rows<kD>(vc, ROT_ENCODE, vnew, kvdtype, nnew, kD, slots, vp.capacity, static_cast<uint32_t *>(vp.codes),
                    vp.norm, nullptr, nullptr, nullptr, bid - nkb, ss);
  } else if (per_head) {
    const int qh = bid - nkb - nvb;  // query head: group qh / 4, head qh % 4
    kfrag_head<BK, QJL>(kc, q, qdtype, kfrag, kconst, counter, qh / kG, qh % kG, ss);
  } else {
    kfrag_group<BK, QJL>(kc, q, qdtype, kfrag, kconst, counter, bid - nkb - nvb, nullptr);
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
// 32-bit multiply kept as such (an opaque multiplier: a power of two here, which would otherwise
// become a shift on the integer ALU pipe).
__device__ __forceinline__ uint32_t mul_lo(uint32_t x, uint32_t m) {
  uint32_t r;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(m));
  return r;
}

constexpr int kSub = 256;            // tokens per sub-chunk: kCWarps consumer warps x 32 tokens
constexpr int kSubBlk = kSub / 16;   // 16-token blocks per sub-chunk
#ifndef TQ_ATTN_STAGES
#define TQ_ATTN_STAGES 3
#endif
#ifndef TQ_ATTN_MAX_CHUNK
#define TQ_ATTN_MAX_CHUNK 4096
#endif
constexpr int kStagesMax = TQ_ATTN_STAGES;  // staging ring depth (sub-chunks in flight), when it fits
#ifndef TQ_ATTN_PRODUCERS
#define TQ_ATTN_PRODUCERS 3
#endif
constexpr int kCWarps = 8;           // consumer warps
constexpr int kProd = TQ_ATTN_PRODUCERS;  // warps that issue the bulk copies (arrays split among them)
constexpr int kMmaThreads = (kCWarps + kProd) * 32;
constexpr int kMaxChunk = TQ_ATTN_MAX_CHUNK;  // tokens per CTA at most
constexpr int kLgS = 40;             // row stride of a warp's weight array (bank-conflict free)

// Shared-memory carve-up of attend_mma_kernel (bytes): the staging ring, each consumer warp's
// private scratch, the query fragments, the CTA's block slots, the barriers.
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
  // ring depth: three buffers where two CTAs per SM still fit, else two
  static constexpr int NS = kStagesMax * buf <= 90 * 1024 ? kStagesMax : 2;
  // per consumer warp: its 32 tokens' value weights [kG][32] and its two blocks' (plane 2,
  // parity) words [2][kD]
  static constexpr size_t WLG = (size_t)kG * kLgS * 4;
  static constexpr size_t WPER = WLG + (size_t)2 * X1W * 4;
  static constexpr size_t ws = NS * buf;
  static constexpr size_t kf = ws + (size_t)kCWarps * WPER;
  static constexpr size_t vb = kf + (size_t)KPlanes<BK, QJL>::regs * 32 * 4;
  static constexpr int MAXBLK = kMaxChunk / 16;
  static constexpr size_t br = vb + (size_t)MAXBLK * 8;
  // full[NS], empty[NS], the merge barrier, then flags, query constants, merge factors
  static constexpr size_t fl = br + (size_t)(2 * NS + 1) * 8;
  static constexpr size_t total = fl + 8 * 4 + 16 * 4 + kG * 4 + kG * 4;
  static_assert(2 + kProd <= 8, "flag words");
  // the warps' partial states at the end of the range reuse the staging ring
  static_assert((size_t)kCWarps * kG * (kD + 2) * 4 <= NS * buf, "warp partials fit the ring");
  static_assert(buf % 16 == 0 && ws % 16 == 0 && kf % 16 == 0 && vb % 16 == 0, "16-byte aligned regions");
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
    case 2: src = static_cast<const char *>(a.k.norm); doff = SM::kn; per = 16u << a.kn4; sstride = 1 << a.kn4; break;
    case 3: src = static_cast<const char *>(a.v.norm); doff = SM::vn; per = 16u << a.vn4; sstride = 1 << a.vn4; break;
    case 4: src = static_cast<const char *>(a.k.signs); doff = SM::ks; per = 256; sstride = 16; break;
    default: src = static_cast<const char *>(a.k.rnorm); doff = SM::kr; per = 16u << a.kn4; sstride = 1 << a.kn4; break;
  }
}

// Producer warp p's copies of sub-chunk `sc` (blocks [NB sc, NB sc + NB) of the CTA's range) into
// staging buffer `sb`, completing on `bar`: one arrival with the expected bytes of its arrays (plus
// `extra` bytes the caller copies on the same barrier), then the copies.  vb[k] = first slot of the
// CTA's block k or -1; contiguous caches copy the nlead leading valid blocks (consecutive slots)
// with one copy per array, paged caches one copy per valid block.
template <int BK, int BV, bool QJL>
__device__ __forceinline__ void stage_sub(const MmaArgs &a, int sc, const int64_t *vb, int nlead,
                                          unsigned char *sb, uint64_t *bar, unsigned extra, int p) {
  using SM = MmaSmem<BK, BV, QJL>;
  constexpr int NA = StageArrays<QJL>::n;  // producer p copies arrays p, p + kProd, ...
  const int lane = threadIdx.x & 31;
  const int k0 = SM::NB * sc;
  unsigned nvalid;
  if (!a.block_table) {
    int n = nlead - k0;
    nvalid = (unsigned)(n < 0 ? 0 : (n > SM::NB ? SM::NB : n));
  } else {
    nvalid = (unsigned)__popc(__ballot_sync(TQ_FULL_MASK, lane < SM::NB && vb[k0 + lane] >= 0));
  }
  unsigned bytes = extra;
#pragma unroll
  for (int arr = p; arr < NA; arr += kProd) {
    const char *src;
    size_t doff;
    unsigned per;
    int64_t sstride;
    stage_array<BK, BV, QJL>(a, arr, src, doff, per, sstride);
    bytes += per * nvalid;
  }
  if (lane == 0) mbar_expect_arrive(bar, bytes);
  __syncwarp();
  if (!a.block_table) {
#pragma unroll
    for (int arr = p; arr < NA; arr += kProd) {
      const char *src;
      size_t doff;
      unsigned per;
      int64_t sstride;
      stage_array<BK, BV, QJL>(a, arr, src, doff, per, sstride);
      if (lane == 0 && nvalid > 0) bulk_g2s(sb + doff, src + vb[k0] * sstride, per * nvalid, bar);
    }
  } else {
    // one copy per valid block; two arrays per round: lanes 0-15 take the blocks of one array,
    // lanes 16-31 the same blocks of the producer's next array
    static_assert(SM::NB == 16, "16 blocks per sub-chunk: half a warp per array");
    const int bl = lane & 15;
    const int64_t base = vb[k0 + bl];
#pragma unroll
    for (int arr0 = p; arr0 < NA; arr0 += 2 * kProd) {
      const int arr = arr0 + (lane >> 4) * kProd;
      if (arr < NA && base >= 0) {
        const char *src;
        size_t doff;
        unsigned per;
        int64_t sstride;
        stage_array<BK, BV, QJL>(a, arr, src, doff, per, sstride);
        bulk_g2s(sb + doff + (size_t)bl * per, src + base * sstride, per, bar);
      }
    }
  }
}

// One CTA = one (sequence, KV head) and a contiguous range of a.chunk tokens (a multiple of 16).
// Warps kCWarps.. (kProd of them) stream the range into a ring of NS sub-chunk buffers with bulk
// copies (each its share of the arrays);
// every other warp owns 32 tokens (two 16-token blocks) of each sub-chunk and runs the whole
// decode on them with its own running softmax state, so no CTA-wide barrier falls inside the
// loop:
//   1. logits of the 4 query heads (bit-plane u8 x s8 MMAs against the query fragments);
//   2. running maximum and sum of the warp's tokens, value weights W = e^{l - M} ||v|| (Sparse V:
//      W = 0 where the weight is below the threshold, see below), their 16-bit fixed-point
//      fragments with the warp's own scale;
//   3. the value MMAs of both blocks over all 128 coordinates into one set of int32
//      accumulators, folded into fp32 sums rescaled by e^{M_old - M_new}.
// At the end the warps' (m, l, o~) are merged in shared memory into the CTA's partial.
// Sparse V ("TurboQuant+ 深度解析" 第六部分): with a threshold tau > 0 a token's value row is left
// out when e^{l - M} < tau max(1, l_old e^{M_old - M}), a bound that is at least its final softmax
// weight (the running sum only grows and the running maximum's token counts 1), or when
// e^{l - Mc} < tau with Mc the CTA's running maximum of the head over every consumer warp's tokens
// (a lower bound of the final maximum too, shared through one atomic per warp and sub-chunk), so
// every row it drops has a final weight below tau; blocks whose rows are all dropped skip their
// value MMAs.
template <int BK, int BV, bool QJL, bool NH, bool SPV>
__global__ void __launch_bounds__(kMmaThreads, 2)
attend_mma_kernel(TqConsts kc, TqConsts vc, MmaArgs a, const uint32_t *__restrict__ kfrag,
                  const float *__restrict__ kconst, float *__restrict__ part) {
  using KP = KPlanes<BK, QJL>;
  using SM = MmaSmem<BK, BV, QJL>;
  constexpr int NB = SM::NB;
  constexpr int VT = BV == 3 ? 2 : 1;  // value word types: (p0,p1) and (p2, parity)
  extern __shared__ __align__(16) unsigned char smem[];
  const uint4 *kf4 = reinterpret_cast<const uint4 *>(smem + SM::kf);  // [plane][k-step][32]
  int64_t *vball = reinterpret_cast<int64_t *>(smem + SM::vb);       // [MAXBLK] first slot of each block
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::br);      // [SM::NS] copies landed
  uint64_t *empty = full + SM::NS;                                  // [SM::NS] consumers done
  uint64_t *mbar = empty + SM::NS;                                  // the merge's copies
  volatile int *flags = reinterpret_cast<volatile int *>(smem + SM::fl);  // [0] abort, [1] last, [2] issued
  float *kcs = reinterpret_cast<float *>(smem + SM::fl + 32);        // [16] query constants
  float *hM = kcs + 16;                                              // [kG] merge rescale factors
  int *cmax = reinterpret_cast<int *>(hM + kG);  // [kG] CTA running logit maximum (ordered int), Sparse V

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, t = lane & 3;
  const int t0 = s * a.chunk;
  const int64_t grp = (int64_t)b * a.hkv + h;
  const int64_t cap = min(a.k.capacity, a.v.capacity);
  constexpr unsigned FB = KP::regs * 32 * 4;  // the query fragments' bytes

  if (tid == 0) {
    for (int i = 0; i < SM::NS; ++i) {
      mbar_init(&full[i], kProd);
      mbar_init(&empty[i], kCWarps);
    }
    mbar_init(mbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    flags[0] = 0;
    for (int i = 0; i < kProd; ++i) flags[2 + i] = 0;
  }
  // Launched as a programmatic dependent of the query-fragment kernel: everything above overlaps
  // its tail; the caches (appended rows), fragments and counters are read only after this.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  int L = a.seq_lens[b];
  L = L < 0 ? 0 : (L > a.max_len ? a.max_len : L);
  const int t1 = min(L, t0 + a.chunk);
  const int nsub = t1 > t0 ? (t1 - t0 + kSub - 1) / kSub : 0;
  // the CTA's blocks: first slot, or -1 past the sequence or the arrays (contiguous caches: the
  // valid blocks are a prefix, the slots consecutive)
  const int nblk = (t1 - t0 + 15) / 16;
  int nlead = 0;
  if (!a.block_table) {
    const int64_t base0 = grp * a.ctx_stride + t0;
    const int64_t fit = base0 < cap ? (cap - base0) / 16 : 0;
    nlead = (int)(fit < nblk ? fit : nblk);
  }
  for (int i = tid; i < SM::MAXBLK; i += kMmaThreads) {
    int64_t base = -1;
    if (i < nblk) {
      base = token_slot(a, b, h, t0 + 16 * i);
      if (base < 0 || base + 16 > cap) base = -1;
    }
    vball[i] = base;
  }
  if (tid < 16) kcs[tid] = kconst[grp * 16 + tid];
  if constexpr (SPV)
    if (tid < kG) cmax[tid] = ord_float(-INFINITY);
  __syncthreads();

  // consumer state: running maximum and sum of head t (same on every gid of a warp) and the value
  // sums of head t at coordinates 16 gid + i (rotated domain)
  float Mrun = -INFINITY, Lw = 0.f;
  float o[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i] = 0.f;
  // Test hook (tq_debug_wait_probe): one bounded wait on the merge barrier, armed for bytes that
  // no copy sends, so that it runs out while the first sub-chunks' copies are in flight; the CTA
  // then takes the same abort path as a staging timeout (flag, drain its copies, return).
  const int probe = g_tq_wait_probe;
  if (probe > 0 && tid == 0) {
    mbar_expect_arrive(mbar, 16u);
    bool ok = false;
    for (int i = 0; i < probe && !ok; ++i) ok = mbar_try_wait(mbar, 0u);
    if (!ok) flags[0] = 1;
  }

  if (warp >= kCWarps) {
    // ------------------------------------------------------------ producers: the staging ring
    const int pw = warp - kCWarps;
    int sc = 0;
    for (; sc < nsub; ++sc) {
      const int st = sc % SM::NS;
      if (sc >= SM::NS) {
        const bool ok = mbar_wait_bounded(&empty[st], (unsigned)((sc / SM::NS) - 1) & 1u);
        if (!__all_sync(TQ_FULL_MASK, ok) || flags[0]) {
          if (lane == 0) flags[0] = 1;
          break;
        }
      }
      stage_sub<BK, BV, QJL>(a, sc, vball, nlead, smem + (size_t)st * SM::buf, &full[st],
                             (sc == 0 && pw == 0) ? FB : 0u, pw);
      if (sc == 0 && pw == 0 && lane == 0) bulk_g2s(smem + SM::kf, kfrag + grp * KP::regs * 32, FB, &full[0]);
    }
    if (lane == 0) flags[2 + pw] = sc;  // sub-chunks issued
  } else {
    // ------------------------------------------------------------ consumers: 32 tokens each
    unsigned char *wsp = smem + SM::ws + (size_t)warp * SM::WPER;
    float *lgw = reinterpret_cast<float *>(wsp);                       // [kG][kLgS] value weights
    uint32_t *x1w = reinterpret_cast<uint32_t *>(wsp + SM::WLG);       // [2][kD] (plane 2, parity)
    const float tau = a.sparse_v;
    for (int sc = 0; sc < nsub; ++sc) {
      const int st = sc % SM::NS;
      const bool ok = mbar_wait_bounded(&full[st], (unsigned)(sc / SM::NS) & 1u);
      if (!__all_sync(TQ_FULL_MASK, ok) || flags[0]) {
        if (lane == 0) flags[0] = 1;
        break;
      }
      const unsigned char *sb = smem + (size_t)st * SM::buf;
      const uint32_t *skc = reinterpret_cast<const uint32_t *>(sb + SM::kc);
      const uint32_t *sks = reinterpret_cast<const uint32_t *>(sb + SM::ks);
      const unsigned char *skn = sb + SM::kn, *skr = sb + SM::kr;
      const uint32_t *svc = reinterpret_cast<const uint32_t *>(sb + SM::vc);
      const unsigned char *svn = sb + SM::vn;
      const int64_t *vb = vball + NB * sc;  // validity of this sub-chunk's blocks
      const int tk0 = t0 + sc * kSub;

      // ---------------------------------------------------------- 1. logits (tokens x heads)
      // blocks 2w and 2w + 1; the query fragments of one (plane, k-step) serve both.  A = the key
      // words masked in place (bytes 0 or 2^shift; B carries 2^-shift).
      float lgt[2][2], nvk[2][2];
      {
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
          for (int stp = 0; stp < 4; ++stp) {
            const uint4 f = kf4[(P * 4 + stp) * 32 + lane];
            const uint32_t mlo = 0x01010101u << stp, mhi = 0x01010101u << (stp + 4);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
              const uint32_t a0 = w[kb][0][P] & mlo, a1 = w[kb][1][P] & mlo;
              const uint32_t a2 = w[kb][0][P] & mhi, a3 = w[kb][1][P] & mhi;
              mma_u8s8(acc[kb][pt][0], a0, a1, a2, a3, f.x, f.y);
              mma_u8s8(acc[kb][pt][1], a0, a1, a2, a3, f.z, f.w);
            }
          }
        }
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          const int blk = 2 * warp + kb;
          const bool bok = vb[blk] >= 0;
          // the four limbs of each of the two tokens (gid, gid + 8) combined in pairs
          const int i0 = blk * 16 + gid, i1 = i0 + 8;
          float dc0, dc1, sc0, sc1;
          {
            const int (&A)[4] = acc[kb][0][0];
            const int (&B)[4] = acc[kb][0][1];
            fma2((float)A[1], (float)A[3], 256.f, (float)A[0], (float)A[2], dc0, dc1);
            fma2((float)B[0], (float)B[2], 65536.f, dc0, dc1, dc0, dc1);
            fma2((float)B[1], (float)B[3], 16777216.f, dc0, dc1, dc0, dc1);
            fma2(dc0, dc1, kcs[t], -kcs[8 + t], -kcs[8 + t], sc0, sc1);
          }
          if constexpr (QJL) {
            const int (&A)[4] = acc[kb][1][0];
            const int (&B)[4] = acc[kb][1][1];
            float ds0, ds1;
            fma2((float)A[1], (float)A[3], 256.f, (float)A[0], (float)A[2], ds0, ds1);
            fma2((float)B[0], (float)B[2], 65536.f, ds0, ds1, ds0, ds1);
            fma2((float)B[1], (float)B[3], 16777216.f, ds0, ds1, ds0, ds1);
            fma2(ds0, ds1, kcs[4 + t], -kcs[12 + t], -kcs[12 + t], ds0, ds1);
            sc0 = fmaf(kc.qjl_scale * staged_norm<NH>(skr, i0), ds0, sc0);
            sc1 = fmaf(kc.qjl_scale * staged_norm<NH>(skr, i1), ds1, sc1);
          }
          const bool ok0 = bok && tk0 + i0 < t1, ok1 = bok && tk0 + i1 < t1;
          lgt[kb][0] = ok0 ? a.scale * staged_norm<NH>(skn, i0) * sc0 : -INFINITY;
          lgt[kb][1] = ok1 ? a.scale * staged_norm<NH>(skn, i1) * sc1 : -INFINITY;
          nvk[kb][0] = ok0 ? staged_norm<NH>(svn, i0) : 0.f;  // masked slots may hold stale bytes
          nvk[kb][1] = ok1 ? staged_norm<NH>(svn, i1) : 0.f;
        }
      }

      // ---------------------------------------------------------- 2. softmax state, weights
      // lane (gid, t) holds head t of tokens gid, gid + 8 of both blocks; lanes sharing t see
      // the same head, so reductions run over gid (xor 4, 8, 16)
      float lmax = fmaxf(fmaxf(lgt[0][0], lgt[0][1]), fmaxf(lgt[1][0], lgt[1][1]));
      float nvmax = fmaxf(fmaxf(nvk[0][0], nvk[0][1]), fmaxf(nvk[1][0], nvk[1][1]));
#pragma unroll
      for (int m = 4; m <= 16; m <<= 1) {
        lmax = fmaxf(lmax, __shfl_xor_sync(TQ_FULL_MASK, lmax, m));
        nvmax = fmaxf(nvmax, __shfl_xor_sync(TQ_FULL_MASK, nvmax, m));
      }
      const float Mnew = fmaxf(Mrun, lmax);
      const float al = Mnew == -INFINITY ? 1.f : __expf(Mrun - Mnew);
      float gate = tau * fmaxf(1.f, Lw * al);  // Sparse V: drop rows with e^{l - M} < gate
      if (SPV && Mnew != -INFINITY) {
        // the CTA's running maximum of head t (every consumer warp's tokens so far) is also at most
        // the final maximum, so a row with e^{l - Mc} < tau has a final weight below tau
        if (gid == 0) atomicMax(&cmax[t], ord_float(Mnew));
        __syncwarp();
        const float Mc = unord_float(cmax[t]);
        gate = fmaxf(gate, tau * __expf(Mc - Mnew));
      }
      float sw = 0.f;
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float l = lgt[kb][r];
          const float wgt = l == -INFINITY ? 0.f : __expf(l - Mnew);
          sw += wgt;
          lgw[t * kLgS + kb * 16 + gid + 8 * r] = (wgt < gate) ? 0.f : wgt * nvk[kb][r];
        }
#pragma unroll
      for (int m = 4; m <= 16; m <<= 1) sw += __shfl_xor_sync(TQ_FULL_MASK, sw, m);
      Lw = fmaf(Lw, al, sw);
      Mrun = Mnew;
      if constexpr (BV == 3) {
        // (plane 2, parity) words of the two blocks, parity = p0 ^ p1 ^ p2: lane computes
        // coordinates 4 lane .. 4 lane + 3 of each block
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint32_t *bw = svc + (2 * warp + kk) * SM::VBW;
          const uint4 A = *reinterpret_cast<const uint4 *>(bw + 4 * lane);
          const uint2 hw2 = *reinterpret_cast<const uint2 *>(bw + kD + 2 * lane);
          const uint32_t A4[4] = {A.x, A.y, A.z, A.w};
          const uint32_t H4[4] = {hw2.x, hw2.x >> 16, hw2.y, hw2.y >> 16};
          uint32_t X4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) X4[e] = __byte_perm(H4[e], A4[e] ^ (A4[e] >> 16) ^ H4[e], 0x5410);
          *reinterpret_cast<uint4 *>(x1w + kk * kD + 4 * lane) = make_uint4(X4[0], X4[1], X4[2], X4[3]);
        }
      }
      __syncwarp();
      // B fragments of the value MMAs.  Lane (gid, t): column = (head gid/2, limb gid&1).  The k
      // index runs over (token, plane) pairs in the order the value words give them: register 0
      // = tokens t, t+8 of the low plane, then of the high plane; register 1 = the same for
      // tokens t+4, t+12.  Byte = limb of X = floor(W 2 e_P sc + dither), dithered so that the
      // many sub-unit tail weights are unbiased rather than all rounded down.
      const int gh = gid >> 1, l = gid & 1;
      float scl, inv;
      weight_scale(nvmax * 2.f * vc.plane_coef_max, scl, inv);
      float C[2 * VT];
#pragma unroll
      for (int P = 0; P < 2 * VT; ++P) C[P] = 2.f * scl * vc.plane_coef[P];
      const uint32_t sel = (uint32_t)l | ((uint32_t)(4 + l) << 4);  // byte l of two words
      const uint32_t key0 = ((uint32_t)grp * (uint32_t)a.max_len + (uint32_t)tk0) * 4u + (uint32_t)gh;
      uint32_t bfr[2][2 * VT];
      bool live[2];
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kb = 2 * warp + kk;
        const float *wr = &lgw[gh * kLgS + kk * 16];
        const int toks[4] = {t, t + 8, t + 4, t + 12};
        float W[4], dz[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          W[i] = wr[toks[i]];
          dz[i] = dither1(key0 + 4u * (uint32_t)(kb * 16 + toks[i]));
        }
        live[kk] = __any_sync(TQ_FULL_MASK, (W[0] > 0.f) | (W[1] > 0.f) | (W[2] > 0.f) | (W[3] > 0.f));
#pragma unroll
        for (int x = 0; x < VT; ++x)
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int i0 = 2 * rr, i1 = 2 * rr + 1;  // the two tokens of this register
            uint32_t x0, x1, x2, x3;
            fma_floor2(W[i0], W[i1], C[2 * x], dz[i0], dz[i1], x0, x1);
            fma_floor2(W[i0], W[i1], C[2 * x + 1], dz[i0], dz[i1], x2, x3);
            bfr[kk][2 * x + rr] = __byte_perm(__byte_perm(x0, x1, sel), __byte_perm(x2, x3, sel), 0x5410);
          }
      }

      // ---------------------------------------------------------- 3. value sum, all coordinates
      // m-tile mt: row gid <-> coordinate 16 gid + 2 mt, row gid + 8 <-> 16 gid + 2 mt + 1.
      // Token bits t, t+8 (and t+4, t+12) of both planes of a word are moved to bit 7 of each byte
      // by a multiply (the FMA pipe) and kept by one AND: bytes 0 or 128.
      int accv[8][4];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int z = 0; z < 4; ++z) accv[mt][z] = 0;
      // the codebook's constant term uses the same integers: one more MMA per fragment pair with
      // every A byte 128 gives 128 sum X of head t in limbs c0 (low), c1 (high) of lane (gid, t)
      int accc[4] = {0, 0, 0, 0};
      const uint32_t mlo = 1u << (7 - t), mhi = 1u << (3 - t);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kb = 2 * warp + kk;
        if (!live[kk] || vb[kb] < 0) continue;
#pragma unroll
        for (int x = 0; x < VT; ++x) {
          mma_u8u8(accc, 0x80808080u, 0x80808080u, 0x80808080u, 0x80808080u, bfr[kk][2 * x], bfr[kk][2 * x + 1]);
          const uint32_t *src = (x == 0) ? svc + kb * SM::VBW + 16 * gid : x1w + kk * kD + 16 * gid;
          uint32_t X[16];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 u = *reinterpret_cast<const uint4 *>(src + 4 * q);
            X[4 * q] = u.x; X[4 * q + 1] = u.y; X[4 * q + 2] = u.z; X[4 * q + 3] = u.w;
          }
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            const uint32_t r0 = X[2 * mt], r1 = X[2 * mt + 1];
            const uint32_t a0 = mul_lo(r0, mlo) & 0x80808080u, a1 = mul_lo(r1, mlo) & 0x80808080u;
            const uint32_t a2 = mul_lo(r0, mhi) & 0x80808080u, a3 = mul_lo(r1, mhi) & 0x80808080u;
            mma_u8u8(accv[mt], a0, a1, a2, a3, bfr[kk][2 * x], bfr[kk][2 * x + 1]);
          }
        }
      }
      // accv[mt]: c0/c1 = (coordinate 16 gid + 2 mt, head t, limb 0/1), c2/c3 = (+1, ...):
      // 128 sum_tok X b; with s = 2b - 1 the codebook's constant term is -(1/2) sum X
      const float cterm = 0.5f * fmaf(256.f, (float)accc[1], (float)accc[0]);  // 64 sum X
      const float ct2 = -cterm * inv;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        float v0, v1, u0, u1;
        fma2((float)accv[mt][1], (float)accv[mt][3], 256.f, (float)accv[mt][0], (float)accv[mt][2], v0, v1);
        fma2(v0, v1, inv, ct2, ct2, u0, u1);
        fma2(o[2 * mt], o[2 * mt + 1], al, u0, u1, o[2 * mt], o[2 * mt + 1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive1(&empty[st]);
    }
  }
  __syncthreads();
  if (flags[0]) {
    // a wait gave up: report, give the copies still in flight a bounded time to land (they write
    // this CTA's shared memory), and leave without writing partials
    if (tid == 0) {
      atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
      int issued = 0;
      for (int i = 0; i < kProd; ++i) issued = max(issued, flags[2 + i]);
      for (int sc = issued > SM::NS ? issued - SM::NS : 0; sc < issued; ++sc)
        mbar_wait_bounded(&full[sc % SM::NS], (unsigned)(sc / SM::NS) & 1u);
    }
    __syncthreads();
    return;
  }

  // ---------------------------------------------------------------- the CTA's partials
  // every copy has been consumed: the warps' states go through the ring, then one (m, l, o~) per
  // head is formed from them with their log-sum-exp weights
  constexpr int WR = kD + 2;
  float *wst = reinterpret_cast<float *>(smem);  // [kCWarps][kG][WR]: m, l, o~
  if (warp < kCWarps) {
    float *row = wst + (warp * kG + t) * WR;
#pragma unroll
    for (int i = 0; i < 16; ++i) row[2 + 16 * gid + i] = o[i];
    if (gid == 0) {
      row[0] = Mrun;
      row[1] = Lw;
    }
  }
  __syncthreads();
  for (int i = tid; i < kG * kD; i += kMmaThreads) {
    const int g = i / kD, j = i % kD;
    float Mx = -INFINITY;
#pragma unroll
    for (int w2 = 0; w2 < kCWarps; ++w2) Mx = fmaxf(Mx, wst[(w2 * kG + g) * WR]);
    float v = 0.f, lsum = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < kCWarps; ++w2) {
      const float *row = wst + (w2 * kG + g) * WR;
      const float f = row[0] == -INFINITY ? 0.f : __expf(row[0] - Mx);
      v = fmaf(f, row[2 + j], v);
      lsum = fmaf(f, row[1], lsum);
    }
    const int64_t pb = (((int64_t)b * a.hq + (int64_t)h * kG + g) * a.splits + s) * (kD + 4);
    part[pb + 2 + j] = v;
    if (j == 0) {
      part[pb] = Mx;
      part[pb + 1] = lsum;
    }
  }
  if (a.out == nullptr) return;

  // ---------------------------------------------------------------- merge (last CTA of the group)
  // The last CTA of this (sequence, KV head) to finish merges the splits of its 4 heads with
  // their log-sum-exp weights and undoes the rotation once:
  //   o = D_V (1/sqrt d) H (sum_s e^{m_s - M} o~_s) / (sum_s e^{m_s - M} l_s).
  // release: the barrier orders every thread's partial stores before thread 0's fence, which
  // (cumulatively) orders them before the count at device scope
  __syncthreads();
  volatile int *last = flags + 1;
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
    if (tid == 0) mbar_expect_arrive(mbar, (unsigned)(kG * n * PR * 4));
    __syncthreads();
    if (tid < kG)
      bulk_g2s(stg + (size_t)tid * n * PR, part + pg + ((int64_t)tid * a.splits + s0) * PR, (unsigned)(n * PR * 4),
               mbar);
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
    if (!__syncthreads_and(mbar_wait_bounded(mbar, (unsigned)(s0 / nb) & 1u))) {
      if (tid == 0) {
        atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
        mbar_wait_bounded(mbar, (unsigned)(s0 / nb) & 1u);
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
  // norms in fp16 (both roles; mixed storage takes the general path) or fp32; the Sparse V gate
  // over the CTA's running maximum only in the variant launched with a threshold
  auto kern = a.sparse_v > 0.f ? (a.kn4 == 1 ? attend_mma_kernel<BK, BV, QJL, true, true>
                                             : attend_mma_kernel<BK, BV, QJL, false, true>)
                               : (a.kn4 == 1 ? attend_mma_kernel<BK, BV, QJL, true, false>
                                             : attend_mma_kernel<BK, BV, QJL, false, false>);
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: the grid may start while the preceding kernel on the stream
  // (the query-fragment or decode-prep kernel) finishes; the kernel waits for it before use.  With
  // per-kernel profiling on, an event sits between the two kernels and a plain launch is used.
  if (tq_prof_on()) {
    kern<<<grid, kMmaThreads, smem, st>>>(kc, vc, a, kfrag, kconst, part);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kMmaThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, kc, vc, a, kfrag, kconst, part);
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
  if (kc.norm16 != vc.norm16) return false;  // one norm storage for both roles
  // the norm arrays are copied in bulk: 16-byte aligned bases
  auto a16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(desc.k.norm) || !a16(desc.v.norm) || (kc.m > 0 && !a16(desc.k.rnorm))) return false;
  return true;
}

int attn_fast_chunk(const tq_attn_desc &desc) {
  // Tokens per CTA (a multiple of 16): the 16-token blocks of all (sequence, KV head) rows split
  // evenly over two resident CTAs per SM, so that a uniform batch runs as one full wave; at least
  // one sub-chunk (256 tokens) and at most kMaxChunk (long or ragged batches then run as several
  // waves that the block scheduler balances).
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
  const int64_t lo = kSub / 16, hi = kMaxChunk / 16;
  per = per < lo ? lo : (per > hi ? hi : per);
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
  a.sparse_v = desc.sparse_v > 0.f ? desc.sparse_v : 0.f;
  a.kn4 = kc.norm16 ? 1 : 2;
  a.vn4 = vc.norm16 ? 1 : 2;
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
  // one block per query head while that keeps the launch under one block per SM, else per group
  const int groups = batch * a.hkv;
  const int per_head = batch * a.hq <= tq_sm_count() ? 1 : 0;
  const unsigned grid0 = (unsigned)(nkb + nvb + (per_head ? batch * a.hq : groups));
  // small launches stage S in each block's shared memory (all of it requested at once); large
  // ones read its transposed copy from L1 / L2 so that many blocks fit on an SM
  const size_t fsm = (QJL && per_head) ? sizeof(float) * kD * (kD + 4) : 0;
  if (fsm) {
    cudaError_t e0 = tq_smem_limit(reinterpret_cast<const void *>(decode_prep_kernel<BK, QJL>), (int)fsm);
    if (e0 != cudaSuccess) return e0;
  }
  tq_prof_begin(TQK_DECODE_PREP, st);
  decode_prep_kernel<BK, QJL><<<grid0, kThreads, fsm, st>>>(kc, vc, knew, vnew, kvdtype, nnew, slots, a.k, a.v, q,
                                                            qdtype, kfrag, kconst, a.counter, nkb, nvb, per_head);
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
  a.sparse_v = desc.sparse_v > 0.f ? desc.sparse_v : 0.f;
  a.kn4 = kc.norm16 ? 1 : 2;
  a.vn4 = vc.norm16 ? 1 : 2;
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
