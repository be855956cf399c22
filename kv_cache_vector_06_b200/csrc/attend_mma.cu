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
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct MmaArgs {
  int hq, hkv, max_len, chunk, splits, block_size, max_blocks;
  int64_t ctx_stride;
  float scale;
  const int32_t *seq_lens;
  const int32_t *block_table;
  tq_packed k, v;
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
  return (float)((x * 2654435769u) >> 8) * (1.0f / 16777216.0f);
}

__device__ __forceinline__ int64_t token_slot(const MmaArgs &a, int b, int h, int t) {
  if (a.block_table) {
    const int blk = a.block_table[(int64_t)b * a.max_blocks + t / a.block_size];
    return blk < 0 ? -1 : ((int64_t)blk * a.hkv + h) * a.block_size + t % a.block_size;
  }
  return ((int64_t)b * a.hkv + h) * a.ctx_stride + t;
}

// Signed byte limbs of v = l0 + 2^8 l1 + 2^16 l2 + 2^24 l3, each l in [-128, 127].
__device__ __forceinline__ int next_limb(int &v) {
  const int l = ((v + 128) & 255) - 128;
  v = (v - l) >> 8;
  return l;
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
  static constexpr int regs = all * 4 * 2 * 2;          // planes x k-steps x n-tiles x regs
};

// Query-side B fragments of the logit MMAs for one (sequence, KV head): for plane P, k-step s,
// n-tile nt, register r and lane (gid, t): bytes i = 0..3 hold limb (gid & 1) + 2 nt of
//   round(X_P[head gid/2][32 t + s + 4 r + 8 i] * 2^(F - s - 4 r)),
// X_P = 2 e_P q' (code planes, parity), 2 p (sign plane); F per head and part so that
// |X| 2^F <= 2^30.  kconst: 2^-F_code, 2^-F_sign, (sum e_P) sum q', sum p per head.
template <int BK, bool QJL>
__device__ __forceinline__ void kfrag_group(const TqConsts &kc, const void *__restrict__ q, int dtype,
                                            uint32_t *__restrict__ kfrag, float *__restrict__ kconst, int grp,
                                            float *sS) {
  using KP = KPlanes<BK, QJL>;
  __shared__ float qs[kG][kD];           // q', the rotated queries
  __shared__ float X[KP::all][kG][kD];
  __shared__ float red[kG][4];
  __shared__ int fexp[kG][2];
  // grp = b * hkv + h; its query heads are rows grp * 4 + g
  const int tid = threadIdx.x;
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
    stage_rows_padded(sS, kc.S, kD, kD);
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
      fexp[g][0] = mc > 0.f ? 30 - ec : 0;
      fexp[g][1] = ms > 0.f ? 30 - es : 0;
      red[g][0] = ldexpf(1.f, -fexp[g][0]);
      red[g][1] = ldexpf(1.f, -fexp[g][1]);
      red[g][2] = kc.plane_coef_sum * sq;
      red[g][3] = sp;
    }
  }
  __syncthreads();
  if (tid < 16) kconst[(int64_t)grp * 16 + tid] = red[tid % 4][tid / 4];
  uint32_t *out = kfrag + (int64_t)grp * KP::regs * 32;
  for (int idx = tid; idx < KP::regs * 32; idx += kThreads) {
    const int ln = idx & 31;
    int rest = idx >> 5;
    const int r = rest & 1;
    rest >>= 1;
    const int nt = rest & 1;
    rest >>= 1;
    const int s = rest & 3;
    const int P = rest >> 2;
    const int gid = ln >> 2, t = ln & 3;
    const int g = gid >> 1, limb = (gid & 1) + 2 * nt;
    const int shift = s + 4 * r;
    const int F = fexp[g][(QJL && P == KP::code) ? 1 : 0];
    uint32_t word = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = 32 * t + s + 4 * r + 8 * i;
      int v = __float2int_rn(ldexpf(X[P][g][j], F - shift));
      int l = 0;
#pragma unroll
      for (int k = 0; k <= 3; ++k) {
        const int li = next_limb(v);
        if (k == limb) l = li;
      }
      word |= (uint32_t)(l & 255) << (8 * i);
    }
    out[idx] = word;
  }
}

template <int BK, bool QJL>
__global__ void __launch_bounds__(kThreads)
kfrag_kernel(TqConsts kc, const void *__restrict__ q, int dtype, uint32_t *__restrict__ kfrag,
             float *__restrict__ kconst) {
  extern __shared__ __align__(16) float sS[];
  kfrag_group<BK, QJL>(kc, q, dtype, kfrag, kconst, blockIdx.x, sS);
}

// One launch for the work that precedes the split kernel in a decode step: blocks
// [0, nkb) append-encode the new keys (8 per block, fused QJL projection), blocks [nkb, nkb + nvb)
// the new values, and the remaining blocks build one (sequence, KV head)'s query fragments.  The
// three jobs are independent, so their latencies overlap instead of adding up.
template <int BK, bool QJL>
__global__ void __launch_bounds__(kThreads)
decode_prep_kernel(TqConsts kc, TqConsts vc, const void *__restrict__ knew, const void *__restrict__ vnew,
                   int kvdtype, int64_t nnew, const int64_t *__restrict__ slots, tq_packed kp, tq_packed vp,
                   const void *__restrict__ q, int qdtype, uint32_t *__restrict__ kfrag,
                   float *__restrict__ kconst, int nkb, int nvb) {
  extern __shared__ __align__(16) float sS[];
  const int bid = blockIdx.x;
  if (bid < nkb) {
    rotate_rows<kD>(kc, ROT_ENCODE, knew, kvdtype, nnew, kD, slots, kp.capacity, static_cast<uint32_t *>(kp.codes),
                    kp.norm, kp.rnorm, nullptr, QJL ? static_cast<uint32_t *>(kp.signs) : nullptr, bid, sS);
  } else if (bid < nkb + nvb) {
    rotate_rows<kD>(vc, ROT_ENCODE, vnew, kvdtype, nnew, kD, slots, vp.capacity, static_cast<uint32_t *>(vp.codes),
                    vp.norm, nullptr, nullptr, nullptr, bid - nkb, sS);
  } else {
    kfrag_group<BK, QJL>(kc, q, qdtype, kfrag, kconst, bid - nkb - nvb, sS);
  }
}

// 16-byte asynchronous global -> shared copy (zero-fill when `ok` is false).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool ok) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  const int n = ok ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(sa), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

// Shared-memory carve-up of attend_mma_kernel (bytes).
template <int BK, int BV, bool QJL, int CH>
struct MmaSmem {
  static constexpr int NBLK = CH / 16;
  static constexpr int KCW = BK * 4;                // K code words per key
  static constexpr int KSW = QJL ? 4 : 0;           // K sign words per key
  static constexpr int VBW = BV * kD / 2;           // V words per 16-token block
  static constexpr int X1W = BV == 3 ? kD : 0;      // (plane 2, parity) words per block
  static constexpr size_t kc = 0;
  static constexpr size_t ks = kc + (size_t)CH * KCW * 4;
  static constexpr size_t kn = ks + (size_t)CH * KSW * 4;
  static constexpr size_t kr = kn + (size_t)CH * 4;
  static constexpr size_t vc = kr + (size_t)CH * 4;
  static constexpr size_t vn = vc + (size_t)NBLK * VBW * 4;
  static constexpr size_t x1 = vn + (size_t)CH * 4;
  static constexpr size_t lg = x1 + (size_t)NBLK * X1W * 4;
  static constexpr size_t vf = lg + (size_t)kG * CH * 4;
  static constexpr size_t vb = vf + (size_t)NBLK * 32 * 16;
  static constexpr size_t st = vb + (size_t)NBLK * 8;
  static constexpr size_t total = st + 256;
  static_assert((size_t)4 * kG * kD * 4 <= st, "the value-sum buffer reuses the staging area");
};

template <int BK, int BV, bool QJL, int CH>
__global__ void __launch_bounds__(kThreads, 1)
attend_mma_kernel(TqConsts kc, TqConsts vc, MmaArgs a, const uint32_t *__restrict__ kfrag,
                  const float *__restrict__ kconst, float *__restrict__ part) {
  using KP = KPlanes<BK, QJL>;
  using SM = MmaSmem<BK, BV, QJL, CH>;
  constexpr int NBLK = SM::NBLK;
  constexpr int KB_PER_WARP = NBLK / kWarps;
  constexpr int VT = BV == 3 ? 2 : 1;  // value word types: (p0,p1) and (p2, parity)
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t *skc = reinterpret_cast<uint32_t *>(smem + SM::kc);
  uint32_t *sks = reinterpret_cast<uint32_t *>(smem + SM::ks);
  float *skn = reinterpret_cast<float *>(smem + SM::kn);
  float *skr = reinterpret_cast<float *>(smem + SM::kr);
  uint32_t *svc = reinterpret_cast<uint32_t *>(smem + SM::vc);
  float *svn = reinterpret_cast<float *>(smem + SM::vn);
  uint32_t *sx1 = reinterpret_cast<uint32_t *>(smem + SM::x1);
  float *lg = reinterpret_cast<float *>(smem + SM::lg);          // [kG][CH] logits, then weights
  uint4 *vfrag = reinterpret_cast<uint4 *>(smem + SM::vf);       // [NBLK][32]
  int64_t *vbase = reinterpret_cast<int64_t *>(smem + SM::vb);   // [NBLK]
  float *hstat = reinterpret_cast<float *>(smem + SM::st);       // [4][kG]
  int *wsum16 = reinterpret_cast<int *>(smem + SM::st) + 4 * kG; // [kG]
  float *obuf = reinterpret_cast<float *>(smem + SM::kc);        // [4][kG][kD], after phase 3's loop

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, t = lane & 3;
  int L = a.seq_lens[b];
  L = L < 0 ? 0 : (L > a.max_len ? a.max_len : L);
  const int t0 = s * CH;
  const int t1 = min(L, t0 + CH);
  const int64_t grp = (int64_t)b * a.hkv + h;
  const int64_t cap = min(a.k.capacity, a.v.capacity);

  // ---------------------------------------------------------------- stage 0: the chunk into smem
  if (tid < NBLK) {
    const int tb = t0 + 16 * tid;
    const int64_t base = tb < t1 ? token_slot(a, b, h, tb) : -1;  // a 16-slot block start
    vbase[tid] = (base >= 0 && base + 16 <= cap) ? base : -1;
  }
  __syncthreads();
  {
    // one loop per array; granules are 16 bytes, blocks are 16 consecutive slots
    const char *kcodes = static_cast<const char *>(a.k.codes);
    const char *vcodes = static_cast<const char *>(a.v.codes);
    constexpr int GK = BK * 16, GV = BV * 16;
    for (int idx = tid; idx < NBLK * GK; idx += kThreads) {
      const int kb = idx / GK, g = idx - kb * GK;
      const int64_t base = vbase[kb];
      cp_async16(reinterpret_cast<char *>(skc) + (size_t)idx * 16,
                 kcodes + (base >= 0 ? base : 0) * (SM::KCW * 4) + 16 * g, base >= 0);
    }
    for (int idx = tid; idx < NBLK * GV; idx += kThreads) {
      const int kb = idx / GV, g = idx - kb * GV;
      const int64_t base = vbase[kb];
      cp_async16(reinterpret_cast<char *>(svc) + (size_t)idx * 16,
                 vcodes + ((base >= 0 ? base : 0) >> 4) * (SM::VBW * 4) + 16 * g, base >= 0);
    }
    if constexpr (QJL) {
      const char *ksigns = static_cast<const char *>(a.k.signs);
      for (int idx = tid; idx < NBLK * 16; idx += kThreads) {
        const int kb = idx >> 4, g = idx & 15;
        const int64_t base = vbase[kb];
        cp_async16(reinterpret_cast<char *>(sks) + (size_t)idx * 16,
                   ksigns + (base >= 0 ? base : 0) * 16 + 16 * g, base >= 0);
      }
    }
    {
      // norms: 4 granules per block for ||k||, ||v|| (and gamma with QJL)
      constexpr int NA = QJL ? 3 : 2;
      for (int idx = tid; idx < NBLK * 4 * NA; idx += kThreads) {
        const int arr = idx / (NBLK * 4), rem = idx - arr * (NBLK * 4);
        const int kb = rem >> 2, g = rem & 3;
        const int64_t base = vbase[kb];
        const float *src = arr == 0 ? a.k.norm : (arr == 1 ? a.v.norm : a.k.rnorm);
        float *dst = arr == 0 ? skn : (arr == 1 ? svn : skr);
        cp_async16(dst + rem * 4, src + (base >= 0 ? base : 0) + 4 * g, base >= 0);
      }
    }
    cp_async_wait_all();
  }
  __syncthreads();

  // ---------------------------------------------------------------- phase 1: logits (keys x heads)
  {
    uint32_t kb[KP::all][4][2][2];
    const uint32_t *fr = kfrag + grp * KP::regs * 32 + lane;
#pragma unroll
    for (int P = 0; P < KP::all; ++P)
#pragma unroll
      for (int st = 0; st < 4; ++st)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int r = 0; r < 2; ++r) kb[P][st][nt][r] = fr[((((P * 4 + st) * 2 + nt) * 2) + r) * 32];
    const float cfc = kconst[grp * 16 + t], cfs = kconst[grp * 16 + 4 + t];
    const float cq = kconst[grp * 16 + 8 + t], cp = kconst[grp * 16 + 12 + t];
#pragma unroll 1
    for (int mb = 0; mb < KB_PER_WARP; ++mb) {
      const int blk = warp * KB_PER_WARP + mb;
      uint32_t w[2][KP::all];
      bool ok[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = blk * 16 + gid + 8 * r;
        ok[r] = vbase[blk] >= 0 && t0 + i < t1;
#pragma unroll
        for (int P = 0; P < BK; ++P) w[r][P] = skc[i * SM::KCW + P * 4 + t];
        if constexpr (BK == 3) w[r][3] = w[r][0] ^ w[r][1] ^ w[r][2];
        if constexpr (QJL) w[r][KP::code] = sks[i * SM::KSW + t];
      }
      int acc[2][2][4];
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 2; ++y)
#pragma unroll
          for (int z = 0; z < 4; ++z) acc[x][y][z] = 0;
#pragma unroll
      for (int P = 0; P < KP::all; ++P) {
        const int pt = (QJL && P == KP::code) ? 1 : 0;
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          const uint32_t mlo = 0x01010101u << st, mhi = 0x01010101u << (st + 4);
          const uint32_t a0 = w[0][P] & mlo, a1 = w[1][P] & mlo, a2 = w[0][P] & mhi, a3 = w[1][P] & mhi;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) mma_u8s8(acc[pt][nt], a0, a1, a2, a3, kb[P][st][nt][0], kb[P][st][nt][1]);
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = blk * 16 + gid + 8 * r;
        const float dc = (float)acc[0][0][2 * r] + 256.f * (float)acc[0][0][2 * r + 1] +
                         65536.f * (float)acc[0][1][2 * r] + 16777216.f * (float)acc[0][1][2 * r + 1];
        float sc = fmaf(dc, cfc, -cq);
        if constexpr (QJL) {
          const float ds = (float)acc[1][0][2 * r] + 256.f * (float)acc[1][0][2 * r + 1] +
                           65536.f * (float)acc[1][1][2 * r] + 16777216.f * (float)acc[1][1][2 * r + 1];
          sc = fmaf(kc.qjl_scale * skr[i], fmaf(ds, cfs, -cp), sc);
        }
        lg[t * CH + i] = ok[r] ? a.scale * skn[i] * sc : -INFINITY;
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- phase 2: softmax weights
  if (warp < kG) {
    // warp g: max logit, weights w = e^{l - max}, W = w * ||v||, sum w, max W for head g
    const int g = warp;
    float mx = -INFINITY;
    for (int i = lane; i < CH; i += 32) mx = fmaxf(mx, lg[g * CH + i]);
    mx = warp_max_f(mx);
    float sw = 0.f, mW = 0.f;
    for (int i = lane; i < CH; i += 32) {
      const float l = lg[g * CH + i];
      const float wgt = l == -INFINITY ? 0.f : __expf(l - mx);
      const float W = wgt * svn[i];
      lg[g * CH + i] = W;
      sw += wgt;
      mW = fmaxf(mW, W);
    }
    sw = warp_sum_f(sw);
    mW = warp_max_f(mW);
    if (lane == 0) {
      int e = 0;
      frexpf(mW, &e);  // mW < 2^e, so mW * 2^(15 - e) + 1 < 2^16
      const int F = mW > 0.f ? 15 - e : 0;
      hstat[0 * kG + g] = mx;
      hstat[1 * kG + g] = sw;
      hstat[2 * kG + g] = ldexpf(1.f, F);
      hstat[3 * kG + g] = ldexpf(1.f, -F);
      wsum16[g] = 0;
    }
  } else if constexpr (BV == 3) {
    // warps 4-7: (plane 2, parity) words, parity = p0 ^ p1 ^ p2, once per block and coordinate
    for (int idx = tid - kG * 32; idx < NBLK * kD; idx += kThreads - kG * 32) {
      const int kb = idx / kD, j = idx % kD;
      const uint32_t A = svc[kb * SM::VBW + j];
      const uint32_t hw = svc[kb * SM::VBW + kD + (j >> 1)] >> (16 * (j & 1));
      const uint32_t par = (A ^ (A >> 16) ^ hw) & 0xffffu;
      sx1[kb * SM::X1W + j] = (hw & 0xffffu) | (par << 16);
    }
  }
  __syncthreads();
  {
    // B fragments of the value MMAs: lane (gid, t) = column (head gid/2, plane gid&1) and
    // tokens t, t+8 (register 0) and t+4, t+12 (register 1); n-tile = limb.
    const int g = gid >> 1, ps = gid & 1;
    const float mul = hstat[2 * kG + g];
    const uint32_t key0 = (uint32_t)((grp * a.splits + s) * CH) * 4u + (uint32_t)g;
    int mine = 0;
    for (int kb = warp; kb < NBLK; kb += kWarps) {
      const float *wr = &lg[g * CH + kb * 16];
      const int toks[4] = {t, t + 8, t + 4, t + 12};
      uint32_t v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t key = key0 + 4u * (uint32_t)(kb * 16 + toks[i]);
        v[i] = (uint32_t)__float2int_rd(fmaf(wr[toks[i]], mul, dither(key)));
      }
      if (ps == 0) mine += (int)(v[0] + v[1] + v[2] + v[3]);
      const int sh = 16 * ps;
      vfrag[kb * 32 + lane] = make_uint4(((v[0] & 255u) | ((v[1] & 255u) << 8)) << sh,
                                         ((v[2] & 255u) | ((v[3] & 255u) << 8)) << sh,
                                         ((v[0] >> 8) | ((v[1] >> 8) << 8)) << sh,
                                         ((v[2] >> 8) | ((v[3] >> 8) << 8)) << sh);
    }
    mine += __shfl_xor_sync(TQ_FULL_MASK, mine, 1);  // lanes t and t^1 share a head and plane
    mine += __shfl_xor_sync(TQ_FULL_MASK, mine, 2);
    if (t == 0 && ps == 0) atomicAdd(&wsum16[g], mine);
  }
  __syncthreads();

  // ---------------------------------------------------------------- phase 3: value sum
  // warp w: coordinate half ch = w & 1 (64 coordinates = 4 m-tiles) and block group w >> 1.
  // In m-tile mt, row gid <-> coordinate 64 ch + 8 gid + 2 mt and row gid + 8 <-> the next one.
  const int ch = warp & 1, bgrp = warp >> 1;
  const int jb = 64 * ch + 8 * gid;
  int accv[4][VT][2][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int x = 0; x < VT; ++x)
#pragma unroll
      for (int y = 0; y < 2; ++y)
#pragma unroll
        for (int z = 0; z < 4; ++z) accv[mt][x][y][z] = 0;
  for (int kb = bgrp; kb < NBLK; kb += 4) {
    if (vbase[kb] < 0) continue;
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
        const uint32_t r0 = X[x][2 * mt], r1 = X[x][2 * mt + 1];
        const uint32_t a0 = (r0 >> t) & 0x01010101u, a1 = (r1 >> t) & 0x01010101u;
        const uint32_t a2 = (r0 >> (t + 4)) & 0x01010101u, a3 = (r1 >> (t + 4)) & 0x01010101u;
        mma_u8u8(accv[mt][x][0], a0, a1, a2, a3, fb.x, fb.y);
        mma_u8u8(accv[mt][x][1], a0, a1, a2, a3, fb.z, fb.w);
      }
  }
  // accv[mt][x][limb][c]: c0/c1 = (coordinate jb + 2 mt, head t, plane lo/hi), c2/c3 = (+1, ...)
  __syncthreads();  // every warp is done with the staged data that obuf overwrites
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float v = 0.f;
#pragma unroll
      for (int x = 0; x < VT; ++x)
#pragma unroll
        for (int ps = 0; ps < 2; ++ps) {
          const float D = (float)accv[mt][x][0][2 * r + ps] + 256.f * (float)accv[mt][x][1][2 * r + ps];
          v = fmaf(2.f * vc.plane_coef[2 * x + ps], D, v);
        }
      obuf[(bgrp * kG + t) * kD + jb + 2 * mt + r] = v;
    }
  __syncthreads();
  for (int i = tid; i < kG * kD; i += kThreads) {
    const int g = i / kD, j = i % kD;
    const float v = obuf[(0 * kG + g) * kD + j] + obuf[(1 * kG + g) * kD + j] + obuf[(2 * kG + g) * kD + j] +
                    obuf[(3 * kG + g) * kD + j];
    const int64_t pb = (((int64_t)b * a.hq + (int64_t)h * kG + g) * a.splits + s) * (kD + 2);
    part[pb + 2 + j] = (v - vc.plane_coef_sum * (float)wsum16[g]) * hstat[3 * kG + g];
  }
  if (tid < kG) {
    const int64_t pb = (((int64_t)b * a.hq + (int64_t)h * kG + tid) * a.splits + s) * (kD + 2);
    part[pb] = hstat[0 * kG + tid];
    part[pb + 1] = hstat[1 * kG + tid];
  }
}

template <int BK, int BV, bool QJL, int CH>
cudaError_t launch_mma(const TqConsts &kc, const TqConsts &vc, const MmaArgs &a, dim3 grid,
                       const uint32_t *kfrag, const float *kconst, float *part, cudaStream_t st) {
  const size_t smem = MmaSmem<BK, BV, QJL, CH>::total;
  cudaError_t e = cudaFuncSetAttribute(attend_mma_kernel<BK, BV, QJL, CH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attend_mma_kernel<BK, BV, QJL, CH><<<grid, kThreads, smem, st>>>(kc, vc, a, kfrag, kconst, part);
  return cudaGetLastError();
}

template <int BK, int BV, bool QJL>
cudaError_t launch_fast(const TqConsts &kc, const TqConsts &vc, const MmaArgs &a, int batch, const void *q,
                        int dtype, uint32_t *kfrag, float *kconst, float *part, cudaStream_t st) {
  const unsigned groups = (unsigned)(batch * a.hkv);
  const size_t fsm = QJL ? sizeof(float) * kD * (kD + 4) : 0;
  if (fsm) {
    cudaError_t e0 = cudaFuncSetAttribute(kfrag_kernel<BK, QJL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsm);
    if (e0 != cudaSuccess) return e0;
  }
  tq_prof_begin(TQK_ATTEND_FRAG, st);
  kfrag_kernel<BK, QJL><<<groups, kThreads, fsm, st>>>(kc, q, dtype, kfrag, kconst);
  tq_prof_end(TQK_ATTEND_FRAG, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)a.splits, (unsigned)a.hkv, (unsigned)batch);
  tq_prof_begin(TQK_ATTEND_SPLIT, st);
  e = a.chunk == 512 ? launch_mma<BK, BV, QJL, 512>(kc, vc, a, grid, kfrag, kconst, part, st)
                     : launch_mma<BK, BV, QJL, 256>(kc, vc, a, grid, kfrag, kconst, part, st);
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
  if (desc.block_table ? (desc.block_size % 16) != 0 : (desc.ctx_stride % 16) != 0) return false;
  return true;
}

int attn_fast_chunk(const tq_attn_desc &desc) {
  // 512-token chunks halve the per-CTA fixed work and the partials to merge; 256 only when
  // 512 would leave fewer than two CTAs per SM
  const int64_t rows = (int64_t)desc.batch * desc.n_kv_heads;
  const int maxlen = desc.max_seq_len > 0 ? desc.max_seq_len : 1;
  const int64_t ctas512 = rows * ((maxlen + 511) / 512);
  return ctas512 >= 2 * 148 ? 512 : 256;
}

size_t attn_fast_extra_bytes(const TqConsts &kc, const tq_attn_desc &desc) {
  const int planes = (kc.bits + (kc.bits == 3 ? 1 : 0)) + (kc.m > 0 ? 1 : 0);
  const int64_t groups = (int64_t)desc.batch * desc.n_kv_heads;
  return (size_t)tq_align_up(groups * planes * 16 * 32 * 4, 256) + (size_t)tq_align_up(groups * 16 * 4, 256);
}

cudaError_t launch_attend_fast(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc,
                               const AttnPlan &plan, const void *q, int dtype, void *extra,
                               float *partials, cudaStream_t st) {
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
  const int nb = (int)((nnew + (kThreads / 32) - 1) / (kThreads / 32));  // one vector per warp (d = 128)
  const unsigned grid0 = (unsigned)(2 * nb + batch * a.hkv);
  const size_t fsm = QJL ? sizeof(float) * kD * (kD + 4) : 0;
  if (fsm) {
    cudaError_t e0 = cudaFuncSetAttribute(decode_prep_kernel<BK, QJL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)fsm);
    if (e0 != cudaSuccess) return e0;
  }
  tq_prof_begin(TQK_DECODE_PREP, st);
  decode_prep_kernel<BK, QJL><<<grid0, kThreads, fsm, st>>>(kc, vc, knew, vnew, kvdtype, nnew, slots, a.k, a.v, q,
                                                            qdtype, kfrag, kconst, nb, nb);
  tq_prof_end(TQK_DECODE_PREP, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)a.splits, (unsigned)a.hkv, (unsigned)batch);
  tq_prof_begin(TQK_ATTEND_SPLIT, st);
  e = a.chunk == 512 ? launch_mma<BK, BV, QJL, 512>(kc, vc, a, grid, kfrag, kconst, part, st)
                     : launch_mma<BK, BV, QJL, 256>(kc, vc, a, grid, kfrag, kconst, part, st);
  tq_prof_end(TQK_ATTEND_SPLIT, st);
  return e;
}
}  // namespace

cudaError_t launch_decode_step_fast(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc,
                                    const AttnPlan &plan, const void *knew, const void *vnew, int kvdtype,
                                    int64_t nnew, const int64_t *slots, const void *q, int qdtype, void *extra,
                                    float *partials, cudaStream_t st) {
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
