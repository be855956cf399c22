// tcgen05 scan for tq_search_topk ("谷歌 TurboQuant 深度拆解" 第三部分 "向量搜索": top-k by the
// estimated inner product ν(⟨q', c[code]⟩ + √(π/2)/m · γ · ⟨p, 2b − 1⟩), score descending then
// index ascending).
//
// The estimate is a contraction of bits with query values (the bit-plane identity of a symmetric
// Lloyd-Max codebook: c = Σ_P e_P s_P (+ e_3 s_0 s_1 s_2 at 3 bits), s_P = 2 bit_P − 1):
//
//   ⟨q', c⟩  = Σ_P Σ_j bit_Pj · 2 e_P q'_j − (Σ_P e_P) Σ_j q'_j
//   ⟨p, 2b−1⟩ = Σ_j b_j · 2 p_j − Σ_j p_j
//
// With many queries this is GEMM-shaped, so it runs on the 5th-generation tensor cores: one
// `tcgen05.mma.kind::i8` per (128 rows, 192 columns, 32 coordinates), A = the rows' plane bits as
// 0/1 bytes (u8) in tensor memory, B = the query values in 24-bit fixed point per query, three
// signed byte limbs (column = limb · 64 + query) in shared memory, int32 accumulators in tensor
// memory (code planes and sign plane apart, 192 columns each).  The int32 sums are exact; the only roundings are the fixed-point
// quantisation of the query values (2^-23 of each query's largest term) and the float combination
// of the limb sums.
//
// A CTA takes 64 queries and one shard of rows, in 128-row blocks.  Warp roles:
//   warps 0-7   expand the rows' packed bits to bytes in tensor memory (two groups of four warps,
//               one row per thread = its lane, alternate planes), one stage = (128 coordinates,
//               plane) = 32 columns, in one of four free 32-column slots;
//   warp 8      allocates tensor memory and issues the MMAs (one thread), committing each stage
//               back to its producers and each block to the epilogue;
//   warp 9      streams the query stages (prepared once per call in the same layout) by bulk copy;
//   warps 10-13 read the accumulators (one row per thread), write the 64 scores to a shared
//               [query][row] tile, release the accumulators, then keep each query's sorted top-k
//               (one warp per query, the tile's rows filtered by the list's k-th entry);
//   warps 14-15 copy the rows' packed words (16 B per row, plane and chunk) into a staging ring
//               with cp.async, so that the expanding threads issue no global loads.
// Every wait is bounded; on a timeout the CTA sets the device flag, drains its own copies and
// MMAs, frees its tensor memory and returns.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "device_common.cuh"
#include "tc_common.cuh"

namespace {

constexpr int kTcQ = 64;                  // queries per CTA
constexpr int kTcN = 3 * kTcQ;            // MMA N: three limbs per query
constexpr int kTcM = 128;                 // rows per block (MMA M)
constexpr int kTcKC = 128;                // coordinates per stage
constexpr int kTcBBytes = kTcN * kTcKC;   // 24 KB of query operand per stage (shared memory)
constexpr int kTcStages = 4;              // A stages live in the four free 32-column tensor-memory slots
constexpr int kTcThreads = 512;
// warp roles
constexpr int kTcWMma = 8, kTcWB = 9, kTcWEpi = 10, kTcWLoad = 14;

// row-word staging ring depth (chunks) for lp stored planes per row
__host__ __device__ constexpr int tc_ring(int lp) { return lp <= 2 ? 8 : 4; }
constexpr int kTcMaxK = 16;
// tensor-memory columns: code sums [0, 192), sign sums [256, 448), A stages at 192, 224, 448, 480
constexpr uint32_t kTcCols = 512;
__host__ __device__ constexpr uint32_t tc_acol(int slot) { return slot < 2 ? 192u + 32u * slot : 448u + 32u * (slot - 2); }

template <int BK, int D>
struct TcShape {
  static constexpr int PL = BK + (BK == 3 ? 1 : 0) + 1;  // code planes (+ parity) + sign plane
  static constexpr int NC = D / kTcKC;                     // stages per plane
  static constexpr int SPB = PL * NC;                      // stages per block
  static constexpr int CODE_BYTES = BK * D / 8;
  static constexpr int SIGN_BYTES = D / 8;
};

struct TcLayout {
  size_t stg, kq, sct, ls, li, bars, slot, total;
  int ns;
};

// lp = stored planes per row (code planes + sign plane)
__host__ __device__ inline TcLayout tc_layout(int k, int ns, int lp) {
  auto up16 = [](size_t x) { return (x + 15) & ~(size_t)15; };
  TcLayout L;
  L.ns = ns;
  L.stg = (size_t)ns * kTcBBytes;                     // [ring][lp][128 rows][16 B]
  L.kq = L.stg + (size_t)tc_ring(lp) * lp * kTcM * 16;
  L.sct = L.kq + kTcQ * 16;                           // block scores [64 q][128 rows] f32
  L.ls = L.sct + (size_t)kTcQ * kTcM * 4;             // per query sorted top-k [64 q][k]
  L.li = L.ls + up16((size_t)kTcQ * k * 4);
  L.bars = L.li + up16((size_t)kTcQ * k * 8);
  L.slot = L.bars + (size_t)(3 * ns + 3 + 2 * tc_ring(lp)) * 8;
  L.total = L.slot + 16;
  return L;
}


// Named barrier 1 over the 128 epilogue threads, returning whether `p` held on all of them.
__device__ __forceinline__ bool epi_all(bool p) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.and.pred po, 1, 128, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)p)
      : "memory");
  return r != 0;
}

// Per query: kq[q] = {2^-Fc, 2^-Fs, (Σ_P e_P) Σ q', Σ p}, F chosen so that |2 e_P q'| 2^Fc and
// |2 p| 2^Fs stay below 2^22 (three balanced signed byte limbs); zeros past nq.  One warp per query.
template <int D>
__global__ void __launch_bounds__(256)
search_tc_scale_kernel(TqConsts c, const float *__restrict__ qr, const float *__restrict__ p, int nq, int nq_pad,
                       float *__restrict__ kq) {
  const int q = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (q >= nq_pad) return;
  float emax = 0.f;
  for (int P = 0; P < 4; ++P) emax = fmaxf(emax, fabsf(c.plane_coef[P]));
  float mc = 0.f, ms = 0.f, sq = 0.f, sp = 0.f;
  if (q < nq) {
    for (int j = lane; j < D; j += 32) {
      const float v = qr[(int64_t)q * D + j], pv = p[(int64_t)q * D + j];
      mc = fmaxf(mc, fabsf(2.f * emax * v));
      ms = fmaxf(ms, fabsf(2.f * pv));
      sq += v;
      sp += pv;
    }
  }
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    mc = fmaxf(mc, __shfl_xor_sync(TQ_FULL_MASK, mc, s));
    ms = fmaxf(ms, __shfl_xor_sync(TQ_FULL_MASK, ms, s));
    sq += __shfl_xor_sync(TQ_FULL_MASK, sq, s);
    sp += __shfl_xor_sync(TQ_FULL_MASK, sp, s);
  }
  if (lane == 0) {
    int ec = 0, es = 0;
    frexpf(mc, &ec);
    frexpf(ms, &es);
    const int Fc = mc > 0.f ? 22 - ec : 0, Fs = ms > 0.f ? 22 - es : 0;
    kq[(int64_t)q * 4 + 0] = pow2i(-Fc);
    kq[(int64_t)q * 4 + 1] = pow2i(-Fs);
    kq[(int64_t)q * 4 + 2] = q < nq ? c.plane_coef_sum * sq : 0.f;
    kq[(int64_t)q * 4 + 3] = q < nq ? sp : 0.f;
  }
}

// Query stages: for tile T and stage j = (chunk cc = j / PL, plane P = j % PL), a 24 KB block holding the B matrix
// [192 columns (limb l, query qi)] x [128 coordinates] in the canonical K-major layout: element
// (n, kk) at (n/8)·1024 + (kk/16)·128 + (n%8)·16 + kk%16.  One thread per (query, 16 coordinates):
// three 16-byte stores, one per limb.  Grid (tiles, SPB).
template <int BK, int D>
__global__ void __launch_bounds__(256)
search_tc_bfrag_kernel(TqConsts c, const float *__restrict__ qr, const float *__restrict__ p, int nq,
                       const float *__restrict__ kq, uint8_t *__restrict__ bst) {
  using TS = TcShape<BK, D>;
  const int tile = blockIdx.x, j = blockIdx.y;
  const int P = j % TS::PL, cc = j / TS::PL;  // chunk-major stages
  const bool sgn = P == TS::PL - 1;
  const float coef = sgn ? 2.f : 2.f * c.plane_coef[P];
  uint8_t *out = bst + ((int64_t)tile * TS::SPB + j) * kTcBBytes;
  for (int task = threadIdx.x; task < kTcQ * 8; task += blockDim.x) {
    const int qi = task >> 3, g = task & 7, q = tile * kTcQ + qi;
    // 2^F from the stored 2^-F (exact powers of two)
    const float sc = 1.f / kq[(int64_t)q * 4 + (sgn ? 1 : 0)];
    uint32_t w[3][4];
#pragma unroll
    for (int i4 = 0; i4 < 4; ++i4) {
      uint32_t b[3][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // K index 16 g + 4 i4 + i of the stage = 32 kw + 4 t + i with kw = g / 2, t = 4 (g % 2) + i4:
        // coordinate 32 kw + 8 i + t (the order the expander writes the row bits in)
        const int jj = kTcKC * cc + 32 * (g >> 1) + 8 * i + 4 * (g & 1) + i4;
        const float x = q < nq ? coef * (sgn ? p[(int64_t)q * D + jj] : qr[(int64_t)q * D + jj]) : 0.f;
        const uint32_t u = (uint32_t)__float2int_rn(x * sc) + 0x80808080u;  // balanced limbs: byte l ^ 0x80
#pragma unroll
        for (int l = 0; l < 3; ++l) b[l][i] = ((u >> (8 * l)) & 0xFFu) ^ 0x80u;
      }
#pragma unroll
      for (int l = 0; l < 3; ++l) w[l][i4] = b[l][0] | (b[l][1] << 8) | (b[l][2] << 16) | (b[l][3] << 24);
    }
#pragma unroll
    for (int l = 0; l < 3; ++l) {
      const int n = l * kTcQ + qi;
      *reinterpret_cast<uint4 *>(out + (n >> 3) * 1024 + g * 128 + (n & 7) * 16) =
          make_uint4(w[l][0], w[l][1], w[l][2], w[l][3]);
    }
  }
}

template <int BK, int D>
__global__ void __launch_bounds__(kTcThreads, 1)
search_tc_kernel(TqConsts c, const uint8_t *__restrict__ bst, const float *__restrict__ kq, int nq, tq_packed db,
                 int64_t n, int k, int64_t rows_per_shard, int shards, int ns, float *__restrict__ cand_s,
                 int64_t *__restrict__ cand_i) {
  using TS = TcShape<BK, D>;
  constexpr int PL = TS::PL, NC = TS::NC, SPB = TS::SPB;
  extern __shared__ __align__(1024) unsigned char smem[];
  constexpr int LP = BK + 1;  // stored planes: code planes + sign plane
  constexpr int kR = tc_ring(LP);
  const TcLayout L = tc_layout(k, ns, LP);
  float *sct = reinterpret_cast<float *>(smem + L.sct);
  float *skq = reinterpret_cast<float *>(smem + L.kq);
  float *ls = reinterpret_cast<float *>(smem + L.ls);        // [64 q][k]
  int64_t *li = reinterpret_cast<int64_t *>(smem + L.li);
  uint64_t *afull = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *bfull = afull + ns, *empty = bfull + ns, *accfull = empty + ns, *accempty = accfull + 1,
           *done = accempty + 1, *rfull = done + 1, *rempty = rfull + kR;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + L.slot);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.slot + 4);

  // the query tiles of a shard are adjacent in launch order (x fastest), so they run at the same
  // time and the shard's rows come from DRAM once, the other tiles reading them from L2
  const int tile = blockIdx.x, shard = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t r_begin = (int64_t)shard * rows_per_shard;
  const int64_t r_end = min(n, r_begin + rows_per_shard);
  const int nblk = r_end > r_begin ? (int)((r_end - r_begin + kTcM - 1) / kTcM) : 0;
  const int64_t nst = (int64_t)nblk * SPB;  // stages this CTA runs

  if (tid == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&afull[i], 4);  // one arrival per warp of the expander group
      mbar_init(&bfull[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accfull, 1);
    mbar_init(accempty, 4);  // one arrival per epilogue warp
    mbar_init(done, 1);
    for (int i = 0; i < kR; ++i) {
      mbar_init(&rfull[i], 64);
      mbar_init(&rempty[i], 8);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kTcWMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(tslot)),
                 "r"(kTcCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  for (int i = tid; i < kTcQ * 4; i += kTcThreads) skq[i] = kq[(int64_t)tile * kTcQ * 4 + i];
  for (int i = tid; i < kTcQ * k; i += kTcThreads) {
    ls[i] = -INFINITY;
    li[i] = INT64_MAX;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp < kTcWMma) {
    // ------------------------------------------------------------ producers: bits -> bytes
    // Stages run chunk-major (for each 128 coordinates: the code planes, the parity plane at
    // 3 bits, the sign plane).  A row's words for one chunk (16 B per stored plane) arrive in the
    // staging ring from the loader warps.  Two groups of four warps (one row per thread, the row
    // being the thread's tensor-memory lane) expand alternate planes of a chunk at the same time.
    const int r = tid & (kTcM - 1), hh = tid >> 7;
    bool ok = true;
    const int64_t nchunks = (int64_t)nblk * NC;
    for (int64_t g = 0; g < nchunks && ok; ++g) {
      const int rs = (int)(g % kR);
      // warp-uniform outcome of the bounded waits (each warp arrives once per barrier phase)
      if (!__all_sync(TQ_FULL_MASK, mbar_wait_bounded(&rfull[rs], (unsigned)(g / kR) & 1u))) {
        ok = false;
        break;
      }
      const int64_t gr = r_begin + (g / NC) * kTcM + r;
      uint4 cur[LP];
      const uint4 *st = reinterpret_cast<const uint4 *>(smem + L.stg) + (size_t)rs * LP * kTcM + r;
#pragma unroll
      for (int P = 0; P < LP; ++P) cur[P] = gr < r_end ? st[P * kTcM] : make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
      if (lane == 0) mbar_arrive1(&rempty[rs]);
      uint4 par = make_uint4(0u, 0u, 0u, 0u);
      if (BK == 3)
        par = make_uint4(cur[0].x ^ cur[1].x ^ cur[2].x, cur[0].y ^ cur[1].y ^ cur[2].y,
                         cur[0].z ^ cur[1].z ^ cur[2].z, cur[0].w ^ cur[1].w ^ cur[2].w);
#pragma unroll
      for (int P = 0; P < PL; ++P) {
        if ((P & 1) != hh) continue;
        const int64_t s = g * PL + P;
        const uint4 wv = P < BK ? cur[P] : (P == PL - 1 ? cur[BK] : par);
        const int slot = (int)(s % ns);
        if (!__all_sync(TQ_FULL_MASK, s < ns || mbar_wait_bounded(&empty[slot], (unsigned)((s / ns) - 1) & 1u))) {
          ok = false;
          break;
        }
        // the row's 128 coordinates as 0/1 bytes, 4 per tensor-memory column of its lane: column
        // 8 k + t holds bits t, t + 8, t + 16, t + 24 of word k (one shift and one mask), so K
        // index 32 k + 4 t + i of the stage is coordinate 32 k + 8 i + t (the query operand is
        // built in the same order)
        const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t o[32];
#pragma unroll
        for (int kw = 0; kw < 4; ++kw)
#pragma unroll
          for (int t = 0; t < 8; ++t) o[8 * kw + t] = (wd[kw] >> t) & 0x01010101u;
        tmem_st32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + tc_acol(slot), o);
        asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive1(&afull[slot]);
      }
    }
    if (!ok) *abort_flag = 1;
  } else if (warp >= kTcWLoad) {
    // ------------------------------------------------------------ row loaders
    // 64 threads, two rows each: 16-byte cp.async of every stored plane of a chunk into the
    // staging ring; each thread's arrival on the ring slot fires when its copies have landed.
    const int lt = tid - 32 * kTcWLoad;
    const uint8_t *codes = static_cast<const uint8_t *>(db.codes);
    const uint8_t *signs = static_cast<const uint8_t *>(db.signs);
    const int64_t nchunks = (int64_t)nblk * NC;
    bool ok = true;
    for (int64_t g = 0; g < nchunks; ++g) {
      const int rs = (int)(g % kR);
      if ((g >= kR && !mbar_wait_bounded(&rempty[rs], (unsigned)((g / kR) - 1) & 1u)) || *abort_flag) {
        ok = false;
        break;
      }
      const int cc = (int)(g % NC);
      unsigned char *st = smem + L.stg + (size_t)rs * LP * kTcM * 16;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = 2 * lt + h;
        const int64_t gr = r_begin + (g / NC) * kTcM + r;
        if (gr < r_end) {
#pragma unroll
          for (int P = 0; P < LP; ++P) {
            const uint8_t *src = (P < BK ? codes + gr * TS::CODE_BYTES + P * (D / 8) : signs + gr * TS::SIGN_BYTES) +
                                 16 * cc;
            cp_async16(st + ((size_t)P * kTcM + r) * 16, src);
          }
        }
      }
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_addr(&rfull[rs]))
                   : "memory");
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");
    if (!ok) *abort_flag = 1;
  } else if (warp == kTcWMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // D s32, A u8, B s8, both K-major, N = 192, M = 128
      const uint32_t idesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(kTcN >> 3) << 17) |
                             ((uint32_t)(kTcM >> 4) << 24);
      const uint32_t sbase = smem_addr(smem);
      int64_t s = 0;
      bool ok = true;
      for (int b = 0; b < nblk && ok; ++b) {
        if (b > 0 && !mbar_wait_bounded(accempty, (unsigned)(b - 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < SPB; ++j, ++s) {
          const int slot = (int)(s % ns);
          const unsigned ph = (unsigned)(s / ns) & 1u;
          if (!mbar_wait_bounded(&afull[slot], ph) || !mbar_wait_bounded(&bfull[slot], ph) || *abort_flag) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int P = j % PL;  // chunk-major stages
          const uint32_t acc = tmem + (P == PL - 1 ? 256u : 0u);
          const bool first = j == 0 || j == PL - 1;
          const uint32_t a0 = tmem + tc_acol(slot), b0 = sbase + (uint32_t)slot * kTcBBytes;
#pragma unroll
          for (int t = 0; t < kTcKC / 32; ++t)
            umma_i8_ta(acc, a0 + 8u * t, umma_desc(b0 + 256u * t, 128u, 1024u), idesc, (first && t == 0) ? 0u : 1u);
          umma_commit(&empty[slot]);
        }
        if (ok) umma_commit(accfull);
      }
      if (!ok) *abort_flag = 1;
      // all MMAs this thread issued have completed before tensor memory is freed
      umma_commit(done);
      mbar_wait_bounded(done, 0u);
    }
    __syncwarp();
  } else if (warp == kTcWB) {
    // ------------------------------------------------------------ query stages
    if (lane == 0) {
      const uint8_t *src = bst + (int64_t)tile * SPB * kTcBBytes;
      int64_t s = 0;
      bool ok = true;
      for (; s < nst; ++s) {
        const int slot = (int)(s % ns);
        if ((s >= ns && !mbar_wait_bounded(&empty[slot], (unsigned)((s / ns) - 1) & 1u)) || *abort_flag) {
          ok = false;
          break;
        }
        mbar_expect_arrive(&bfull[slot], kTcBBytes);
        bulk_g2s(smem + (size_t)slot * kTcBBytes, src + (s % SPB) * kTcBBytes, kTcBBytes, &bfull[slot]);
      }
      if (!ok) {
        *abort_flag = 1;
        // drain the copies still landing in this CTA's shared memory
        for (int64_t u = std::max<int64_t>(0, s - ns); u < s; ++u)
          mbar_wait_bounded(&bfull[u % ns], (unsigned)(u / ns) & 1u);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue: scores and top-k
    // Thread = row for the scores (its tensor-memory lane), written to a [query][row] tile; then
    // warp ew keeps the sorted top-k of queries ew, ew + 4, ..., scanning the tile's 128 rows per
    // query against the list's k-th entry.  Named barrier 1 (the 128 epilogue threads) orders the
    // tile between the two phases.
    const int quarter = warp & 3, ew = warp - kTcWEpi;
    const int row = 32 * quarter + lane;
    const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);
    const int qn = min(kTcQ, nq - tile * kTcQ);
    bool ok = true;
    // this block's norms are loaded before the wait for its accumulators
    int64_t gr = r_begin + row;
    float nrm = 0.f, qg = 0.f;
    if (nblk > 0 && gr < r_end) {
      nrm = ld_norm(db.norm, gr, c.norm16);
      qg = c.qjl_scale * ld_norm(db.rnorm, gr, c.norm16);
    }
    for (int b = 0; b < nblk; ++b) {
      // all four warps go on (the previous block's top-k has finished reading the tile) or all stop
      const bool got = mbar_wait_bounded(accfull, (unsigned)b & 1u) && !*abort_flag;
      if (!epi_all(got)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int qb = 0; qb < kTcQ / 16; ++qb) {
        uint32_t v[3][16];
        float a[16];
        // code sums, then sign sums, of queries 16 qb .. 16 qb + 15 (limb l at column l * 64 + q)
#pragma unroll
        for (int l = 0; l < 3; ++l) tmem_ld16(tl + (uint32_t)(l * kTcQ + 16 * qb), v[l]);
        asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int q = 16 * qb + i;
          const float dc = (float)(int)v[0][i] + 256.f * (float)(int)v[1][i] + 65536.f * (float)(int)v[2][i];
          a[i] = fmaf(dc, skq[4 * q], -skq[4 * q + 2]);
        }
#pragma unroll
        for (int l = 0; l < 3; ++l) tmem_ld16(tl + 256u + (uint32_t)(l * kTcQ + 16 * qb), v[l]);
        asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int q = 16 * qb + i;
          const float ds = (float)(int)v[0][i] + 256.f * (float)(int)v[1][i] + 65536.f * (float)(int)v[2][i];
          sct[q * kTcM + row] = nrm * fmaf(qg, fmaf(ds, skq[4 * q + 1], -skq[4 * q + 3]), a[i]);
        }
      }
      // the accumulators may be overwritten by the next block now
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive1(accempty);
      const int64_t r0 = r_begin + (int64_t)b * kTcM;
      const int nr = (int)min((int64_t)kTcM, r_end - r0);
      gr += kTcM;
      if (b + 1 < nblk && gr < r_end) {
        nrm = ld_norm(db.norm, gr, c.norm16);
        qg = c.qjl_scale * ld_norm(db.rnorm, gr, c.norm16);
      }
      asm volatile("bar.sync 1, 128;\n" ::: "memory");
#pragma unroll 1
      for (int q = ew; q < qn; q += 4) {
        float *Ls = ls + q * k;
        int64_t *Li = li + q * k;
        const float ts = Ls[k - 1];
        const int64_t ti = Li[k - 1];
        // lane l holds rows 4 l .. 4 l + 3
        const float4 v4 = *reinterpret_cast<const float4 *>(sct + q * kTcM + 4 * lane);
        const float sv[4] = {v4.x, v4.y, v4.z, v4.w};
        bool cj[4], any = false;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          cj[j] = 4 * lane + j < nr && tq_better(sv[j], r0 + 4 * lane + j, ts, ti);
          any |= cj[j];
        }
        if (__ballot_sync(TQ_FULL_MASK, any) == 0u) continue;
        float bs = lane < k ? Ls[lane] : -INFINITY;
        int64_t bi = lane < k ? Li[lane] : INT64_MAX;
#pragma unroll
        for (int j = 0; j < 4; ++j) warp_topk_insert(bs, bi, k, sv[j], r0 + 4 * lane + j, cj[j]);
        if (lane < k) {
          Ls[lane] = bs;
          Li[lane] = bi;
        }
        __syncwarp();
      }
    }
    if (!ok) *abort_flag = 1;
  }

  // ------------------------------------------------------------ teardown and the shard's top-k
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kTcWMma) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTcCols)
                              : "memory");
  if (*abort_flag) {
    if (tid == 0) atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
    return;
  }
  if (warp >= kTcWEpi && warp < kTcWEpi + 4) {
    const int ew = warp - kTcWEpi;
    for (int qi = ew; qi < kTcQ; qi += 4) {
      const int q = tile * kTcQ + qi;
      if (q >= nq) break;
      if (lane < k) {
        const int64_t o = ((int64_t)q * shards + shard) * k + lane;
        cand_s[o] = ls[qi * k + lane];
        cand_i[o] = li[qi * k + lane];
      }
    }
  }
}

constexpr size_t kTcSmemPerCta = 232448, kTcSmemOneCta = 120 * 1024;

inline int tc_stages(int k, int lp) {
  int ns = kTcStages;
  while (ns > 2 && tc_layout(k, ns, lp).total > kTcSmemPerCta) --ns;
  return ns;
}

int tc_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, v = 0;
    sms = (cudaGetDevice(&dev) == cudaSuccess &&
           cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
              ? v
              : 148;
  }
  return sms;
}

template <int BK, int D>
cudaError_t launch_tc(const TqConsts &c, int shards, const float *qr, const float *p, int nq, const tq_packed &db,
                      int64_t n, int k, void *ws, float *cand_s, int64_t *cand_i, cudaStream_t st) {
  using TS = TcShape<BK, D>;
  const int tiles = (nq + kTcQ - 1) / kTcQ;
  uint8_t *bst = static_cast<uint8_t *>(ws);
  float *kq = reinterpret_cast<float *>(bst + tq_align_up((int64_t)tiles * TS::SPB * kTcBBytes, 256));
  const int ns = tc_stages(k, BK + 1);
  const TcLayout L = tc_layout(k, ns, BK + 1);
  // more than half an SM's shared memory, so that one CTA (and one 512-column tensor-memory
  // allocation) is resident per SM
  const size_t smem = std::max(L.total, kTcSmemOneCta);
  tq_prof_begin(TQK_SEARCH_SCAN, st);
  search_tc_scale_kernel<D><<<(tiles * kTcQ + 7) / 8, 256, 0, st>>>(c, qr, p, nq, tiles * kTcQ, kq);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    search_tc_bfrag_kernel<BK, D><<<dim3((unsigned)tiles, (unsigned)TS::SPB), 256, 0, st>>>(c, qr, p, nq, kq, bst);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = tq_smem_limit(reinterpret_cast<const void *>(search_tc_kernel<BK, D>), (int)smem);
  if (e == cudaSuccess) {
    const int64_t rows_per_shard = ((n + shards - 1) / shards + kTcM - 1) / kTcM * kTcM;
    search_tc_kernel<BK, D><<<dim3((unsigned)tiles, (unsigned)shards), kTcThreads, smem, st>>>(
        c, bst, kq, nq, db, n, k, rows_per_shard, shards, ns, cand_s, cand_i);
    e = cudaGetLastError();
  }
  tq_prof_end(TQK_SEARCH_SCAN, st);
  return e;
}

}  // namespace

bool search_tc_eligible(const TqConsts &c, int nq, int k) {
  return (c.d == 128 || c.d == 256 || c.d == 512 || c.d == 1024) && c.m == c.d && c.bits >= 1 && c.bits <= 3 &&
         c.fast_ok && c.layout == TQ_LAYOUT_ROWS && k <= kTcMaxK && nq >= kTcQ / 2 &&
         (nq + kTcQ - 1) / kTcQ <= 65535;
}

size_t search_tc_ws_bytes(const TqConsts &c, int nq) {
  const int tiles = (nq + kTcQ - 1) / kTcQ;
  const int pl = c.bits + (c.bits == 3 ? 1 : 0) + 1;
  const int64_t spb = (int64_t)pl * (c.d / kTcKC);
  return (size_t)tq_align_up((int64_t)tiles * spb * kTcBBytes, 256) +
         (size_t)tq_align_up((int64_t)tiles * kTcQ * 16, 256);
}

int search_tc_shards(int nq, int64_t n) {
  // one CTA per SM; cost = waves x (blocks per shard + about two blocks of start-up and merge)
  const int64_t tiles = (nq + kTcQ - 1) / kTcQ, slots = tc_sms();
  const int64_t nb = (n + kTcM - 1) / kTcM;
  const int64_t max_s = std::max<int64_t>(1, std::min<int64_t>(4096, nb / 2));
  int64_t best = 1, best_cost = INT64_MAX;
  for (int64_t s = 1; s <= max_s; ++s) {
    const int64_t waves = (tiles * s + slots - 1) / slots;
    const int64_t cost = waves * ((nb + s - 1) / s + 2);
    if (cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return (int)best;
}

cudaError_t launch_search_tc(const TqConsts &c, int shards, const float *qr, const float *p, int nq,
                             const tq_packed &db, int64_t n, int k, void *ws, float *cand_s, int64_t *cand_i,
                             cudaStream_t st) {
#define TQ_TC(BKV, DV) \
  if (c.bits == BKV && c.d == DV) return launch_tc<BKV, DV>(c, shards, qr, p, nq, db, n, k, ws, cand_s, cand_i, st);
  TQ_TC(1, 128) TQ_TC(2, 128) TQ_TC(3, 128)
  TQ_TC(1, 256) TQ_TC(2, 256) TQ_TC(3, 256)
  TQ_TC(1, 512) TQ_TC(2, 512) TQ_TC(3, 512)
  TQ_TC(1, 1024) TQ_TC(2, 1024) TQ_TC(3, 1024)
#undef TQ_TC
  return cudaErrorInvalidValue;
}

// The device flags of this translation unit's kernels (see tq_device_status).
TQ_DEVICE_FLAGS_ACCESSOR(search_tc_device_flags)
