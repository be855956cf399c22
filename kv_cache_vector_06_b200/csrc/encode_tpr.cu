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

// Codes by the codebook's symmetry.  The thresholds are antisymmetric (t_(L-2-k) = -t_k, the middle
// one 0), so with the H = L/2 - 1 positive ones t+_k and cnt = #{k : |y| >= t+_k}:
//   code = L/2 + cnt                       for y >= 0,
//   code = L/2 - 1 - cnt (= ~cnt mod L/2)    for y < 0 (with > in place of >=),
// the same count as #{i : t_i <= y} (ties go up).  The strict comparison of a negative y is the
// non-strict one on the float just below |y|.  cnt's b - 1 bits come from a binary search over
// the positive thresholds (b - 1 comparisons), each setting bit j of a word of its own; the code's
// bit planes are then the sign word and the count words complemented where y < 0.
template <int BITS>
struct Sym {
  static constexpr int H = (1 << (BITS - 1)) - 1;  // positive thresholds
  static constexpr int HW = H > 0 ? H : 1;
  static constexpr int CW = BITS > 1 ? BITS - 1 : 1;  // count words
};

// One coordinate j (of the NW 32-bit words a thread packs): bit j of the sign word and of the count
// words.
template <int BITS, int NW>
__device__ __forceinline__ void sym_quant(float y, const float (&Tp)[Sym<BITS>::HW], uint32_t (&sw)[NW],
                                          uint32_t (&cw)[Sym<BITS>::CW][NW], int j) {
  const bool pos = y >= 0.f;
  const uint32_t bit = 1u << (j & 31);
  if (pos) sw[j >> 5] |= bit;
  if constexpr (BITS >= 2) {
    const float a = __uint_as_float((__float_as_uint(y) & 0x7fffffffu) - (pos ? 0u : 1u));
    if constexpr (BITS == 2) {
      if (a >= Tp[0]) cw[0][j >> 5] |= bit;
    } else if constexpr (BITS == 3) {
      const bool b1 = a >= Tp[1];
      const bool b0 = a >= (b1 ? Tp[2] : Tp[0]);
      if (b1) cw[1][j >> 5] |= bit;
      if (b0) cw[0][j >> 5] |= bit;
    } else {
      const bool b2 = a >= Tp[3];
      const bool b1 = a >= (b2 ? Tp[5] : Tp[1]);
      const bool b0 = a >= (b2 ? (b1 ? Tp[6] : Tp[4]) : (b1 ? Tp[2] : Tp[0]));
      if (b2) cw[2][j >> 5] |= bit;
      if (b1) cw[1][j >> 5] |= bit;
      if (b0) cw[0][j >> 5] |= bit;
    }
  }
}

// The code's bit planes: plane BITS - 1 is the sign word; the lower planes are the count's bits,
// complemented where y < 0.
template <int BITS, int NW>
__device__ __forceinline__ void sym_planes(const uint32_t (&sw)[NW], const uint32_t (&cw)[Sym<BITS>::CW][NW],
                                           uint32_t (&w)[BITS][NW]) {
#pragma unroll
  for (int q = 0; q < NW; ++q) {
    const uint32_t n = ~sw[q];
    w[BITS - 1][q] = sw[q];
#pragma unroll
    for (int k = 0; k < BITS - 1; ++k) w[k][q] = cw[k][q] ^ n;
  }
}

// 32 x 32 bit transpose across a warp: lane i holds row i (bit j = element (i, j)) and gets back
// column `lane` (bit i = element (i, lane)).  Five exchange stages with the partner lane at
// distance 16, 8, 4, 2, 1: the halves and bytes move by byte permutes, the nibbles, pairs and
// single bits by a rotate of the partner's word and a bit select.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane) {
  uint32_t y = __shfl_xor_sync(TQ_FULL_MASK, x, 16);
  x = __byte_perm(x, y, (lane & 16) ? 0x3276 : 0x5410);
  y = __shfl_xor_sync(TQ_FULL_MASK, x, 8);
  x = __byte_perm(x, y, (lane & 8) ? 0x3715 : 0x6240);
#pragma unroll
  for (int s = 4; s >= 1; s >>= 1) {
    const uint32_t m = s == 4 ? 0x0F0F0F0Fu : (s == 2 ? 0x33333333u : 0x55555555u);
    y = __shfl_xor_sync(TQ_FULL_MASK, x, s);
    const bool hi = (lane & s) != 0;
    const uint32_t keep = hi ? ~m : m;
    const uint32_t r = __funnelshift_r(y, y, hi ? s : 32 - s);
    x = (x & keep) | (r & ~keep);
  }
  return x;
}

struct TprArgs {
  const char *x;
  int64_t ld_bytes;
  int64_t n;
  const int64_t *slots;  // ROWS layout only (NULL: slot = row)
  int64_t capacity;
  uint32_t *codes;
  void *norm, *rnorm;  // fp32 or fp16 (TqConsts::norm16)
  uint32_t *signs;       // structured QJL only
};

// Token-block layout: the 32 rows of a warp, rows [wrow0, wrow0 + 32), are two 16-slot blocks
// (slot = row).  A bit transpose of each plane word gives lane j coordinate 32 g + j of all 32
// rows, i.e. its word of both blocks.  Only whole blocks are written (the caller passes a
// multiple of 16 rows).  Called by all lanes of the warp.
template <int BITS>
__device__ __forceinline__ void store_blk16(const TqConsts &c, const TprArgs &a, const uint32_t (&w)[BITS][kTD / 32],
                                            int64_t wrow0, int lane) {
  if (wrow0 >= a.n) return;  // uniform over the warp
  const bool twoblk = wrow0 + 16 < a.n;
  uint32_t *blkA = a.codes + (wrow0 >> 4) * (int64_t)(16 * c.code_words);
  uint32_t *blkB = blkA + 16 * c.code_words;
#pragma unroll
  for (int q2 = 0; q2 < BITS / 2; ++q2)
#pragma unroll
    for (int g = 0; g < kTD / 32; ++g) {
      const uint32_t lo = warp_transpose32(w[2 * q2][g], lane), hi = warp_transpose32(w[2 * q2 + 1][g], lane);
      blkA[q2 * kTD + 32 * g + lane] = __byte_perm(lo, hi, 0x5410);
      if (twoblk) blkB[q2 * kTD + 32 * g + lane] = __byte_perm(lo, hi, 0x7632);
    }
  if constexpr (BITS & 1) {
    // the odd last plane packs coordinates 2 j' (bits 0-15) and 2 j' + 1 (bits 16-31): lane j'
    // takes them from the transposed words of coordinates 64 g .. 64 g + 63
#pragma unroll
    for (int g = 0; g < kTD / 64; ++g) {
      const uint32_t ta = warp_transpose32(w[BITS - 1][2 * g], lane);
      const uint32_t tb = warp_transpose32(w[BITS - 1][2 * g + 1], lane);
      const int se = (2 * lane) & 31;
      const uint32_t ea = __shfl_sync(TQ_FULL_MASK, ta, se), eb = __shfl_sync(TQ_FULL_MASK, tb, se);
      const uint32_t oa = __shfl_sync(TQ_FULL_MASK, ta, se + 1), ob = __shfl_sync(TQ_FULL_MASK, tb, se + 1);
      const uint32_t ev = lane < 16 ? ea : eb, od = lane < 16 ? oa : ob;
      blkA[(BITS / 2) * kTD + 32 * g + lane] = __byte_perm(ev, od, 0x5410);
      if (twoblk) blkB[(BITS / 2) * kTD + 32 * g + lane] = __byte_perm(ev, od, 0x7632);
    }
  }
}

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
  // the positive thresholds (codes by symmetry), or all of them where the residual is formed
  constexpr int NT = SRHT ? L - 1 : Sym<BITS>::HW;
  float thr[NT];
#pragma unroll
  for (int i = 0; i < (SRHT ? L - 1 : Sym<BITS>::H); ++i) thr[i] = c.thresholds[SRHT ? i : L / 2 + i];
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
    float T[NT];
#pragma unroll
    for (int i = 0; i < (SRHT ? L - 1 : Sym<BITS>::H); ++i) T[i] = thr[i] * scl;
    uint32_t w[BITS][kTD / 32];
    float rr = 0.f;
    if constexpr (SRHT) {
      // the plain count, whose code feeds the residual (fewer live registers than the
      // thermometer words here)
#pragma unroll
      for (int P = 0; P < BITS; ++P)
#pragma unroll
        for (int q = 0; q < kTD / 32; ++q) w[P][q] = 0u;
#pragma unroll
      for (int j = 0; j < kTD; ++j) {
        int code = 0;
#pragma unroll
        for (int i = 0; i < L - 1; ++i) code += v[j] >= T[i] ? 1 : 0;
#pragma unroll
        for (int P = 0; P < BITS; ++P) w[P][j >> 5] |= (uint32_t)((code >> P) & 1) << (j & 31);
        const float r = fmaf(v[j], inv, -cen[code]);  // residual, rotated domain
        v[j] = r;
        rr = fmaf(r, r, rr);
      }
    } else {
      uint32_t sw[kTD / 32], tw[Sym<BITS>::CW][kTD / 32];
#pragma unroll
      for (int q = 0; q < kTD / 32; ++q) {
        sw[q] = 0u;
#pragma unroll
        for (int k = 0; k < Sym<BITS>::CW; ++k) tw[k][q] = 0u;
      }
#pragma unroll
      for (int j = 0; j < kTD; ++j) sym_quant<BITS, kTD / 32>(v[j], T, sw, tw, j);
      sym_planes<BITS, kTD / 32>(sw, tw, w);
    }
    if constexpr (BLK) {
      store_blk16<BITS>(c, a, w, tile * kTRows + 32 * warp, lane);
      if (valid) st_norm(a.norm, row, nu, c.norm16);
    } else {
      const int64_t slot = valid ? (a.slots ? a.slots[row] : row) : -1;
      if (valid && slot >= 0 && slot < a.capacity) {
        uint4 *dst = reinterpret_cast<uint4 *>(a.codes + slot * c.code_words);
        // b planes of 4 words = the row's b * 16 bytes (code_words = 4 b at d = 128)
#pragma unroll
        for (int P = 0; P < BITS; ++P) dst[P] = make_uint4(w[P][0], w[P][1], w[P][2], w[P][3]);
        st_norm(a.norm, slot, nu, c.norm16);
        if constexpr (SRHT) {
          // structured QJL: z = H (D2 r), the first m signs
          st_norm(a.rnorm, slot, sqrtf(rr), c.norm16);
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


// ------------------------------------------------------------------ bf16 rows on tcgen05
// bf16 rows: the rotation runs on the tensor cores.  With B[n][k] = (-1)^popcount(n & k) D_k
// (entries +-1, exact in bf16), y = H (D x) = X B^T is one 128 x 128 x 128 bf16 MMA with fp32
// accumulation per tile of 128 rows: the sums the butterflies form, added in another order.  The
// norm follows from ||y|| = sqrt(d) ||x||, and the thresholds are scaled by ||y||.
//
// Keys with a dense Gaussian JL matrix (m = d = 128) then form z = S r on the tensor cores as three
// TF32 products (r_hi S_hi + r_hi S_lo + r_lo S_hi, each operand split as x = head + (x - head),
// the head being x with its low 13 mantissa bits cleared; the dropped r_lo S_lo term is below
// 2^-20 of the products), which keeps z within about 2^-20 of the fp32 dot product's scale:
//   A = the tile's residual rows, written by their own threads into tensor memory (lane = row,
//       one column per coordinate): r_hi for the first two products, then r_lo in the same
//       columns for the third;
//   B = S_hi, S_lo in shared memory (canonical K-major layout, staged once per CTA);
//   D = z in tensor memory, read back by the row's thread for its sign bits.
//
// Two groups of eight compute warps take alternate tiles, each with its own staging buffer and
// tensor-memory columns (y, later the residual; with QJL also z).  Warps w and w + 4 of a group
// see the same 32 tensor-memory lanes (rows), so each row is shared by two threads: one per half
// of the 128 columns (half the registers of a whole row, twice the warps).  The two halves of a
// row's sums of squares are added through shared memory in a fixed order.  Warp 16 issues the
// MMAs (one thread) and owns the allocation.  The MMA thread issues a tile's rotation before the
// other group's products, so that one group's rotation is not queued behind them, and a group
// packs its previous tile's signs before it encodes its next tile.
// The staged tile: bf16 (r, k) at (k / 8) 2048 + 16 r + 2 (k % 8), i.e. each K chunk of 8
// elements holds all 128 rows contiguously (core matrices of 8 rows x 16 bytes).
constexpr int kQGroups = 2;
constexpr int kQWarps = 8;                                 // compute warps per group
constexpr int kQGThreads = kQWarps * 32;
constexpr int kQThreads = (kQWarps * kQGroups + 1) * 32;
constexpr int kQMmaWarp = kQWarps * kQGroups;
constexpr int kHalf = kTD / 2;                             // columns per compute thread
constexpr int kHW = kHalf / 32;                            // plane words per compute thread
constexpr uint32_t kXLbo = 2048, kXSbo = 128;   // bf16 tiles (rows and the rotation)
constexpr uint32_t kQLbo = 128, kQSbo = 4096;   // S: (n, k) at (n / 8) 4096 + (k / 4) 128 + 16 (n % 8) + 4 (k % 4)
constexpr int kXBytes = kTRows * kTD * 2;      // one staged bf16 tile
constexpr int kQSBytes = kTD * kTD * 4;        // one of S_hi / S_lo

template <bool QJL>
struct TcSmem {
  static constexpr size_t x = 0;                                  // [group] staged tile
  static constexpr size_t rot = x + (size_t)kQGroups * kXBytes;    // B of the rotation
  static constexpr size_t shi = rot + kXBytes;
  static constexpr size_t slo = shi + (QJL ? kQSBytes : 0);
  static constexpr size_t xch = slo + (QJL ? kQSBytes : 0);       // [group][half][row] partial sums
  static constexpr size_t bars = xch + (size_t)kQGroups * 2 * kTRows * 4;
  // per group: xfull, yfull, yfree, rhi, hidone, rlo, zfull; then done
  static constexpr int NB = 7;
  static constexpr size_t total = bars + (size_t)(NB * kQGroups + 1) * 8;
  static_assert(rot % 1024 == 0 && shi % 1024 == 0, "descriptor base alignment");
};
enum { kBxFull = 0, kByFull, kByFree, kBrHi, kBhiDone, kBrLo, kBzFull };

// Issue the cp.async copies of tile rows [r0, r0 + 128) into the canonical layout (rows past n are
// skipped), by the 256 threads of one group: lane = row within 32 consecutive rows, so that each
// warp's 16-byte writes are contiguous in shared memory.
__device__ __forceinline__ void tc_stage_x(const char *__restrict__ x, int64_t ld_bytes, int64_t n, int64_t r0,
                                           unsigned char *dst, int gi) {
#pragma unroll 4
  for (int cc = gi; cc < kTRows * 16; cc += kQGThreads) {
    const int row = cc & (kTRows - 1), col = cc >> 7;
    if (r0 + row < n) cp_async16(dst + col * kXLbo + row * 16, x + (r0 + row) * ld_bytes + col * 16);
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

__device__ __forceinline__ bool qwait(uint64_t *bar, unsigned parity, volatile int *abort_flag) {
  for (int i = 0; i < (1 << 22); ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  return false;
}

__device__ __forceinline__ void group_sync(int g) {
  if (g == 0)
    asm volatile("bar.sync 1, 256;\n" ::: "memory");
  else
    asm volatile("bar.sync 2, 256;\n" ::: "memory");
}

// True on every thread of group g when `fail` holds on any of its 256 threads (a barrier with an
// OR reduction), so that the group leaves its loop as one and no warp is left at a group barrier.
__device__ __forceinline__ bool group_any(int g, bool fail) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, 256, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)fail), "r"(g + 1)
      : "memory");
  return r != 0;
}

// The group's copies have landed: make them visible to the tensor cores and signal the MMA thread.
__device__ __forceinline__ void tc_x_ready(int g, uint64_t *xfull, int gi) {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  group_sync(g);
  if (gi == 0) mbar_arrive1(xfull);
}

// A thread's half row of z (tensor memory, 64 fp32 columns from `zaddr`): sign words 2 h, 2 h + 1.
// Bit e of a word is set when z >= 0: the words are built from the sign bits, one funnel shift per
// element (m = (m << 1) | sign, last element first) and one complement at the end.  A negative zero
// sum counts as negative here; such a z lies far inside any rounding band around 0.
__device__ __forceinline__ void pack_signs_half(uint32_t zaddr, const TqConsts &c, const TprArgs &a, int64_t slot,
                                                int h) {
  uint32_t sb[kHW];
#pragma unroll
  for (int q = 0; q < kHW; ++q) {
    uint32_t z0[16], z1[16];
    tmem_ld16(zaddr + 32u * q, z0);
    tmem_ld16(zaddr + 32u * q + 16u, z1);
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
    uint32_t m = 0u;
#pragma unroll
    for (int e = 15; e >= 0; --e) m = __funnelshift_l(z1[e], m, 1);
#pragma unroll
    for (int e = 15; e >= 0; --e) m = __funnelshift_l(z0[e], m, 1);
    sb[q] = ~m;
  }
  if (slot >= 0) *reinterpret_cast<uint2 *>(a.signs + slot * c.sign_words + kHW * h) = make_uint2(sb[0], sb[1]);
}

// store_blk16 for the half of the coordinates [64 h, 64 h + 64) whose plane words a warp holds.
template <int BITS>
__device__ __forceinline__ void store_blk16_half(const TqConsts &c, const TprArgs &a, const uint32_t (&w)[BITS][kHW],
                                                 int64_t wrow0, int lane, int h) {
  if (wrow0 >= a.n) return;  // uniform over the warp
  const bool twoblk = wrow0 + 16 < a.n;
  uint32_t *blkA = a.codes + (wrow0 >> 4) * (int64_t)(16 * c.code_words);
  uint32_t *blkB = blkA + 16 * c.code_words;
#pragma unroll
  for (int q2 = 0; q2 < BITS / 2; ++q2)
#pragma unroll
    for (int gg = 0; gg < kHW; ++gg) {
      const int g = kHW * h + gg;
      const uint32_t lo = warp_transpose32(w[2 * q2][gg], lane), hi = warp_transpose32(w[2 * q2 + 1][gg], lane);
      blkA[q2 * kTD + 32 * g + lane] = __byte_perm(lo, hi, 0x5410);
      if (twoblk) blkB[q2 * kTD + 32 * g + lane] = __byte_perm(lo, hi, 0x7632);
    }
  if constexpr (BITS & 1) {
    // odd last plane: coordinates 64 h .. 64 h + 63, two per word
    const uint32_t ta = warp_transpose32(w[BITS - 1][0], lane);
    const uint32_t tb = warp_transpose32(w[BITS - 1][1], lane);
    const int se = (2 * lane) & 31;
    const uint32_t ea = __shfl_sync(TQ_FULL_MASK, ta, se), eb = __shfl_sync(TQ_FULL_MASK, tb, se);
    const uint32_t oa = __shfl_sync(TQ_FULL_MASK, ta, se + 1), ob = __shfl_sync(TQ_FULL_MASK, tb, se + 1);
    const uint32_t ev = lane < 16 ? ea : eb, od = lane < 16 ? oa : ob;
    blkA[(BITS / 2) * kTD + 32 * h + lane] = __byte_perm(ev, od, 0x5410);
    if (twoblk) blkB[(BITS / 2) * kTD + 32 * h + lane] = __byte_perm(ev, od, 0x7632);
  }
}

template <int BITS, bool QJL, bool BLK>
__global__ void __launch_bounds__(kQThreads, 1)
encode_tc_kernel(TqConsts c, TprArgs a) {
  using SM = TcSmem<QJL>;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float cen[TQ_MAX_LEVELS];
  __shared__ uint32_t tslot;
  __shared__ int abort_flag_s;
  volatile int *abort_flag = &abort_flag_s;
  uint64_t *gb = reinterpret_cast<uint64_t *>(smem + SM::bars);  // [group][SM::NB]
  uint64_t *done = gb + SM::NB * kQGroups;
  float *xch = reinterpret_cast<float *>(smem + SM::xch);       // [group][half][row]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int L = 1 << BITS;
  constexpr uint32_t kCols = QJL ? 512u : 256u;  // per group: y / residual (128) [, z (128)]
  constexpr uint32_t kGCols = kCols / kQGroups;

  // B of the rotation: (n, k) = (-1)^popcount(n & k) D_k as bf16, at (k / 8) 2048 + 16 n + 2 (k % 8)
  for (int idx = tid; idx < kTD * kTD; idx += kQThreads) {
    const int n = idx / kTD, k = idx % kTD;
    const bool neg = ((__popc(n & k) & 1) != 0) != (c.signs[k] < 0.f);
    *reinterpret_cast<uint16_t *>(smem + SM::rot + (k >> 3) * kXLbo + n * 16 + (k & 7) * 2) =
        neg ? (uint16_t)0xBF80u : (uint16_t)0x3F80u;
  }
  if constexpr (QJL) {
    // S_hi and S_lo in the canonical K-major layout
    for (int idx = tid; idx < kTD * kTD; idx += kQThreads) {
      const int n = idx / kTD, k = idx % kTD;
      const float sv = c.S[idx];
      const uint32_t hi = tf32_head(sv);
      const float lo = sv - __uint_as_float(hi);
      const uint32_t off = (uint32_t)(n >> 3) * kQSbo + (uint32_t)(k >> 2) * kQLbo + (uint32_t)(n & 7) * 16 +
                           (uint32_t)(k & 3) * 4;
      *reinterpret_cast<uint32_t *>(smem + SM::shi + off) = hi;
      *reinterpret_cast<uint32_t *>(smem + SM::slo + off) = __float_as_uint(lo);
    }
  }
  if (tid < TQ_MAX_LEVELS) cen[tid] = c.centroids[tid];
  if (tid == 0) {
    for (int g = 0; g < kQGroups; ++g) {
      uint64_t *b = gb + SM::NB * g;
      mbar_init(&b[kBxFull], 1);
      mbar_init(&b[kByFull], 1);
      mbar_init(&b[kByFree], kQWarps);
      mbar_init(&b[kBrHi], kQWarps);
      mbar_init(&b[kBhiDone], 1);
      mbar_init(&b[kBrLo], kQWarps);
      mbar_init(&b[kBzFull], 1);
    }
    mbar_init(done, 1);
    abort_flag_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kQMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(&tslot)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // B operands visible to the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  const int64_t ntiles = (a.n + kTRows - 1) / kTRows;
  const int64_t mytiles = ntiles > blockIdx.x ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp == kQMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // rotation: D f32, A and B bf16, both K-major, N = M = 128; products: A and B tf32
      const uint32_t idesc_r = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTD >> 3) << 17) |
                               ((uint32_t)(kTRows >> 4) << 24);
      const uint32_t idesc_q = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kTD >> 3) << 17) |
                               ((uint32_t)(kTRows >> 4) << 24);
      const uint32_t xs = smem_addr(smem + SM::x), rs = smem_addr(smem + SM::rot);
      const uint32_t shi = smem_addr(smem + SM::shi), slo = smem_addr(smem + SM::slo);
      bool ok = true;
      // the products of local tile t (QJL)
      auto products = [&](int64_t t) -> bool {
        const int g = (int)(t % kQGroups);
        const unsigned ph = (unsigned)((t / kQGroups) & 1);
        uint64_t *b = gb + SM::NB * g;
        const uint32_t acol = tmem + kGCols * g, zcol = acol + 128u;
        if (!qwait(&b[kBrHi], ph, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int pass = 0; pass < 2; ++pass)  // r_hi S_hi, r_hi S_lo
#pragma unroll
          for (int ks = 0; ks < kTD / 8; ++ks)
            umma_tf32_ta(zcol, acol + 8u * ks, umma_desc((pass ? slo : shi) + 2u * kQLbo * ks, kQLbo, kQSbo),
                         idesc_q, (pass == 0 && ks == 0) ? 0u : 1u);
        umma_commit(&b[kBhiDone]);
        if (!qwait(&b[kBrLo], ph, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kTD / 8; ++ks)  // r_lo S_hi
          umma_tf32_ta(zcol, acol + 8u * ks, umma_desc(shi + 2u * kQLbo * ks, kQLbo, kQSbo), idesc_q, 1u);
        umma_commit(&b[kBzFull]);
        return true;
      };
      for (int64_t i = 0; i < mytiles && ok; ++i) {
        const int g = (int)(i % kQGroups);
        const unsigned ph = (unsigned)((i / kQGroups) & 1);
        uint64_t *b = gb + SM::NB * g;
        const uint32_t acol = tmem + kGCols * g;
        if (!qwait(&b[kBxFull], ph, abort_flag)) {
          ok = false;
          break;
        }
        if (i >= kQGroups) {
          // the group's columns are free: its previous residual has been used (QJL) or its
          // previous y has been read (values)
          if (!qwait(&b[QJL ? kBzFull : kByFree], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
        }
        tc_fence_after();
        const uint32_t xg = xs + (uint32_t)g * kXBytes;
#pragma unroll
        for (int ks = 0; ks < kTD / 16; ++ks)
          umma_f16_ss(acol, umma_desc(xg + 2u * kXLbo * ks, kXLbo, kXSbo), umma_desc(rs + 2u * kXLbo * ks, kXLbo, kXSbo),
                      idesc_r, ks == 0 ? 0u : 1u);
        umma_commit(&b[kByFull]);
        if constexpr (QJL)
          if (i >= 1 && !products(i - 1)) ok = false;
      }
      if constexpr (QJL)
        if (ok && mytiles > 0 && !products(mytiles - 1)) ok = false;
      if (!ok) *abort_flag = 1;
      umma_commit(done);  // every MMA this thread issued has completed when `done` fires
      qwait(done, 0u, abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute: half a row per thread
    const int g = warp / kQWarps, gw = warp % kQWarps;  // group, warp within the group
    const int quad = gw & 3, h = gw >> 2;               // lane quadrant (rows), column half
    const int gt = 32 * quad + lane;                    // row within the tile
    const int gi = tid - g * kQGThreads;                // thread within the group
    uint64_t *b = gb + SM::NB * g;
    unsigned char *xbuf = smem + SM::x + (size_t)g * kXBytes;
    float *myx = xch + (g * 2 + h) * kTRows + gt, *otx = xch + g * 2 * kTRows + gt;
    const uint32_t lanes = (uint32_t)(32 * quad) << 16;
    const uint32_t abase = tmem + kGCols * g + lanes + (uint32_t)(kHalf * h), zbase = abase + 128u;
    float thr[Sym<BITS>::HW];  // the positive thresholds (value codes by symmetry)
#pragma unroll
    for (int k = 0; k < Sym<BITS>::H; ++k) thr[k] = c.thresholds[L / 2 + k];
    int64_t prev_slot = -1;
    int64_t j = 0;  // this group's tiles so far
    int64_t i = g;  // local tile index
    if (i < mytiles) {
      tc_stage_x(a.x, a.ld_bytes, a.n, (blockIdx.x + i * gridDim.x) * kTRows, xbuf, gi);
      tc_x_ready(g, &b[kBxFull], gi);
    }
    for (; i < mytiles; i += kQGroups, ++j) {
      const int64_t tile = blockIdx.x + i * gridDim.x;
      bool ok = true;
      if constexpr (QJL) {
        // this group's previous z: its signs first (its columns are then free for this tile)
        if (j > 0) {
          ok = qwait(&b[kBzFull], (unsigned)((j - 1) & 1), abort_flag);
          if (group_any(g, !ok || *abort_flag)) break;
          tc_fence_after();
          pack_signs_half(zbase, c, a, prev_slot, h);
        }
      }
      ok = qwait(&b[kByFull], (unsigned)(j & 1), abort_flag);
      if (group_any(g, !ok || *abort_flag)) break;
      tc_fence_after();
      float v[kHalf];
#pragma unroll
      for (int cb = 0; cb < kHalf / 16; ++cb) {
        uint32_t u[16];
        tmem_ld16(abase + 16u * cb, u);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[16 * cb + e] = __uint_as_float(u[e]);
      }
      asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
      if constexpr (!QJL) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive1(&b[kByFree]);
      }
      // the rotation has read this group's tile: stage its next one
      const bool more = i + kQGroups < mytiles;
      if (more) tc_stage_x(a.x, a.ld_bytes, a.n, (blockIdx.x + (i + kQGroups) * gridDim.x) * kTRows, xbuf, gi);

      const int64_t row = tile * kTRows + gt;
      const bool valid = row < a.n;
      const int64_t slot = valid ? (a.slots ? a.slots[row] : row) : -1;
      const bool store = valid && slot >= 0 && slot < a.capacity;
      // ||y||^2 = d ||x||^2: eight partial sums per half, the halves added in a fixed order
      float ps[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ps[e] = 0.f;
#pragma unroll
      for (int jj = 0; jj < kHalf; ++jj) ps[jj & 7] = fmaf(v[jj], v[jj], ps[jj & 7]);
      *myx = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      group_sync(g);
      const float ssy = otx[0] + otx[kTRows];
      const float ny = sqrtf(ssy);
      const float nu = ny * c.inv_sqrt_d;
      const float scl = ny > 0.f ? ny : 1.f;
      uint32_t w[BITS][kHW];
      if constexpr (QJL) {
        const float inv = ny > 0.f ? 1.f / scl : 0.f;
        float T[L - 1];
#pragma unroll
        for (int k = 0; k < L - 1; ++k) T[k] = c.thresholds[k] * scl;
        float rr = 0.f;
        if constexpr (BITS <= 2) {
          // one or two bits: a thermometer word per threshold (code = the number of thresholds
          // passed) and the centroid selected by the same comparisons; the planes are the count's
          // bits (bit 1 = the middle threshold, bit 0 = the parity of the three)
          float cl[L];
#pragma unroll
          for (int k = 0; k < L; ++k) cl[k] = c.centroids[k];
          uint32_t tw[L - 1][kHW];
#pragma unroll
          for (int k = 0; k < L - 1; ++k)
#pragma unroll
            for (int q = 0; q < kHW; ++q) tw[k][q] = 0u;
#pragma unroll
          for (int jj = 0; jj < kHalf; ++jj) {
            const float y = v[jj];
            const uint32_t bit = 1u << (jj & 31);
            float cc = cl[0];
#pragma unroll
            for (int k = 0; k < L - 1; ++k) {
              const bool ge = y >= T[k];
              if (ge) tw[k][jj >> 5] |= bit;
              cc = ge ? cl[k + 1] : cc;
            }
            const float r = fmaf(y, inv, -cc);
            v[jj] = r;
            rr = fmaf(r, r, rr);
          }
#pragma unroll
          for (int q = 0; q < kHW; ++q) {
            if constexpr (BITS == 1) {
              w[0][q] = tw[0][q];
            } else {
              w[1][q] = tw[1][q];
              w[0][q] = tw[0][q] ^ tw[1][q] ^ tw[2][q];
            }
          }
        } else {
#pragma unroll
          for (int P = 0; P < BITS; ++P)
#pragma unroll
            for (int q = 0; q < kHW; ++q) w[P][q] = 0u;
#pragma unroll
          for (int jj = 0; jj < kHalf; ++jj) {
            int code = 0;
#pragma unroll
            for (int k = 0; k < L - 1; ++k) code += v[jj] >= T[k] ? 1 : 0;
#pragma unroll
            for (int P = 0; P < BITS; ++P) w[P][jj >> 5] |= (uint32_t)((code >> P) & 1) << (jj & 31);
            const float r = fmaf(v[jj], inv, -cen[code]);
            v[jj] = r;
            rr = fmaf(r, r, rr);
          }
        }
        // r_hi -> tensor memory (the columns y came from): the first two products start while the
        // residual norms are exchanged and the codes stored
#pragma unroll
        for (int cb = 0; cb < kHalf / 16; ++cb) {
          uint32_t hv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            hv[e] = tf32_head(v[16 * cb + e]);
            v[16 * cb + e] -= __uint_as_float(hv[e]);  // r_lo from here on (exact in fp32)
          }
          tmem_st16(abase + 16u * cb, hv);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive1(&b[kBrHi]);
        group_sync(g);  // both halves have read the norm partials
        *myx = rr;
        group_sync(g);
        const float rr2 = otx[0] + otx[kTRows];
        if (store) {
          uint32_t *dst = a.codes + slot * c.code_words + kHW * h;
#pragma unroll
          for (int P = 0; P < BITS; ++P) *reinterpret_cast<uint2 *>(dst + 4 * P) = make_uint2(w[P][0], w[P][1]);
          if (h == 0) {
            st_norm(a.norm, slot, nu, c.norm16);
            st_norm(a.rnorm, slot, sqrtf(rr2), c.norm16);
          }
        }
        // r_lo into the same columns once those products have read r_hi
        ok = qwait(&b[kBhiDone], (unsigned)(j & 1), abort_flag);
        if (group_any(g, !ok || *abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int cb = 0; cb < kHalf / 16; ++cb) {
          uint32_t lv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) lv[e] = __float_as_uint(v[16 * cb + e]);
          tmem_st16(abase + 16u * cb, lv);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive1(&b[kBrLo]);
        prev_slot = store ? slot : -1;
      } else {
        float T[Sym<BITS>::HW];
#pragma unroll
        for (int k = 0; k < Sym<BITS>::H; ++k) T[k] = thr[k] * scl;
        uint32_t sw[kHW], tw[Sym<BITS>::CW][kHW];
#pragma unroll
        for (int q = 0; q < kHW; ++q) {
          sw[q] = 0u;
#pragma unroll
          for (int k = 0; k < Sym<BITS>::CW; ++k) tw[k][q] = 0u;
        }
#pragma unroll
        for (int jj = 0; jj < kHalf; ++jj) sym_quant<BITS, kHW>(v[jj], T, sw, tw, jj);
        sym_planes<BITS, kHW>(sw, tw, w);
        if constexpr (BLK) {
          store_blk16_half<BITS>(c, a, w, tile * kTRows + 32 * quad, lane, h);
          if (valid && h == 0) st_norm(a.norm, row, nu, c.norm16);
        } else if (store) {
          uint32_t *dst = a.codes + slot * c.code_words + kHW * h;
#pragma unroll
          for (int P = 0; P < BITS; ++P) *reinterpret_cast<uint2 *>(dst + 4 * P) = make_uint2(w[P][0], w[P][1]);
          if (h == 0) st_norm(a.norm, slot, nu, c.norm16);
        }
      }
      if (more) tc_x_ready(g, &b[kBxFull], gi);
    }
    if constexpr (QJL) {
      // the group's last tile's signs
      if (i >= mytiles && j > 0) {
        const bool ok = qwait(&b[kBzFull], (unsigned)((j - 1) & 1), abort_flag);
        if (__all_sync(TQ_FULL_MASK, ok)) {
          tc_fence_after();
          pack_signs_half(zbase, c, a, prev_slot, h);
        }
      }
    }
    if (i < mytiles && lane == 0) *abort_flag = 1;  // left the loop on a failed wait
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
  if (warp == kQMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kCols) : "memory");
  }
}

template <int BITS, bool QJL, bool BLK>
cudaError_t launch_tc_t(const TqConsts &c, const TprArgs &a, cudaStream_t st) {
  static_assert(TcSmem<QJL>::total + 512 <= 227 * 1024, "the tensor-core encode's shared memory (with its static part)");
  const size_t smem = TcSmem<QJL>::total;
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(encode_tc_kernel<BITS, QJL, BLK>), (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (a.n + kTRows - 1) / kTRows;
  const int64_t sms = tq_sm_count();
  const int64_t grid = ntiles < sms ? ntiles : sms;
  tq_prof_begin(QJL ? TQK_ENCODE_QJL_TC : TQK_ENCODE_ROWS, st);
  encode_tc_kernel<BITS, QJL, BLK><<<(unsigned)grid, kQThreads, smem, st>>>(c, a);
  tq_prof_end(QJL ? TQK_ENCODE_QJL_TC : TQK_ENCODE_ROWS, st);
  return cudaGetLastError();
}

template <bool QJL, bool BLK>
cudaError_t launch_tc_b(const TqConsts &c, const TprArgs &a, cudaStream_t st) {
  switch (c.bits) {
    case 1: return launch_tc_t<1, QJL, BLK>(c, a, st);
    case 2: return launch_tc_t<2, QJL, BLK>(c, a, st);
    case 3: return launch_tc_t<3, QJL, BLK>(c, a, st);
    case 4: return launch_tc_t<4, QJL, BLK>(c, a, st);
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
                              const int64_t *slots, int64_t capacity, uint32_t *codes, void *norm, void *rnorm,
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
  if (c.m > 0 && !c.srht) return launch_tc_b<true, false>(c, a, st);  // bf16 rows only (eligibility)
  if (dtype == TQ_BF16 && !c.srht)
    return c.layout == TQ_LAYOUT_BLOCK16 ? launch_tc_b<false, true>(c, a, st) : launch_tc_b<false, false>(c, a, st);
  return dtype == TQ_F32 ? launch_tpr_dt<TQ_F32>(c, a, st) : launch_tpr_dt<TQ_BF16>(c, a, st);
}
