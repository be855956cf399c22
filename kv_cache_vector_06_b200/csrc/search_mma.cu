// Tensor-core scan for tq_search_topk ("谷歌 TurboQuant 深度拆解" 第三部分 "向量搜索": top-k by the
// estimated inner product ν(⟨q', c[code]⟩ + √(π/2)/m · γ · ⟨p, 2b − 1⟩), ordered by score
// descending then index ascending).
//
// The estimate is the same exact bit-plane identity as the decode attention: a symmetric
// Lloyd-Max codebook is Σ_P e_P s_P (+ e_3 s_0 s_1 s_2 at 3 bits), so every term is a 0/1 bit times
// a query-side value.  Per 16 database rows, 8 queries and 32 coordinates of one plane, one
// m16n8k32 u8×s8 MMA per limb: A = the rows' plane bits moved to bit 7 of each byte (multiply +
// AND: bytes 0 or 128), B = the queries' values 2 e_P q' (or 2 p) in 24-bit fixed point per query,
// three signed byte limbs, one n-tile per limb (column = query), so each thread ends with all
// limbs of its two queries.
//
// Lane t of a warp owns the d/128 consecutive words [t·d/128, (t+1)·d/128) of every plane of a
// row; k-step (g, st) of the MMA covers coordinates 32 (t·d/128 + g) + 8 i + st (+ 4), which the
// query fragments follow.
//
// Scan: a CTA takes 8 queries and one shard of rows, streams the shard through shared memory in
// 128-row blocks (bulk copies on an mbarrier; one or two buffers, one or two CTAs per SM, as the
// shared memory allows).  A warp pair scores 32 rows, each warp over half of the k-steps with two
// m-tiles per query-fragment load, then the pair swaps partial sums and each warp finishes one
// m-tile.  Every warp keeps a sorted top-k per query in shared memory (insertions are rare once
// the lists fill); at the end warp q merges query q's 8 warp lists and writes the shard's
// candidates, which the existing merge kernel reduces.  The shard count balances the waves of
// (query tile, shard) CTAs over the SMs.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "device_common.cuh"

namespace {

constexpr int kSmThreads = 256;
constexpr int kSmQ = 8;     // queries per CTA (one n-tile column each)
constexpr int kSmRB = 128;  // rows per block (8 warps x 16)
constexpr int kSmL = 3;     // limbs per value (24-bit fixed point)

template <int BK, int D>
struct SearchMma {
  static constexpr int PL = BK + (BK == 3 ? 1 : 0) + 1;  // code planes (+ parity) + sign plane
  static constexpr int WPL = D / 128;                      // words per lane per plane
  static constexpr int FRAG_WORDS = PL * WPL * 4 * kSmL * 32 * 2;  // u32 per query tile
  static constexpr int CODE_BYTES = BK * D / 8;            // per row
  static constexpr int SIGN_BYTES = D / 8;
};

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t mul_lo(uint32_t x, uint32_t m) {
  uint32_t r;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(m));
  return r;
}

// Query fragments of one tile of 8 queries: frag[(((P·WPL + g)·4 + st)·3 + l)·32 + lane] = uint2
// with bytes i of .x / .y = limb l of round(X_P[q][32 (WPL t + g) + 8 i + st (+4)] · 2^F), lane =
// (query q = lane/4, t = lane%4), X = 2 e_P q' (code planes, parity) or 2 p (sign plane), F per
// query and part with |X| 2^F < 2^22.  kq[q][4] = 2^-F_code/128, 2^-F_sign/128, e_sum Σq', Σp.
template <int BK, int D>
__global__ void __launch_bounds__(kSmThreads)
search_frag_kernel(TqConsts c, const float *__restrict__ qr, const float *__restrict__ p, int nq,
                   uint2 *__restrict__ frag, float *__restrict__ kq) {
  using SP = SearchMma<BK, D>;
  __shared__ int fexp[kSmQ][2];
  const int tile = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float emax = 0.f;  // largest |e_P| over the code planes (and the parity plane)
  for (int P = 0; P < SP::PL - 1; ++P) emax = fmaxf(emax, fabsf(c.plane_coef[P]));
  // warp q: the F exponents and sums of query q of the tile
  {
    const int q = tile * kSmQ + warp;
    float mc = 0.f, ms = 0.f, sq = 0.f, sp = 0.f;
    if (q < nq) {
      for (int j = lane; j < D; j += 32) {
        const float v = qr[(int64_t)q * D + j];
        mc = fmaxf(mc, fabsf(2.f * emax * v));
        sq += v;
        const float pv = p[(int64_t)q * D + j];
        ms = fmaxf(ms, fabsf(2.f * pv));
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
      fexp[warp][0] = Fc;
      fexp[warp][1] = Fs;
      float *o = kq + ((int64_t)tile * kSmQ + warp) * 4;
      o[0] = pow2i(-Fc - 7);
      o[1] = pow2i(-Fs - 7);
      o[2] = q < nq ? c.plane_coef_sum * sq : 0.f;
      o[3] = q < nq ? sp : 0.f;
    }
  }
  __syncthreads();
  uint2 *out = frag + (int64_t)tile * (SP::FRAG_WORDS / 2);
  for (int idx = tid; idx < SP::FRAG_WORDS / 2; idx += kSmThreads) {
    const int ln = idx & 31;
    int rest = idx >> 5;
    const int l = rest % kSmL;
    rest /= kSmL;
    const int st = rest & 3;
    rest >>= 2;
    const int g = rest % SP::WPL;
    const int P = rest / SP::WPL;
    const int qi = ln >> 2, t = ln & 3;
    const int q = tile * kSmQ + qi;
    const bool sgn = P == SP::PL - 1;
    const float coef = sgn ? 2.f : 2.f * c.plane_coef[P];
    const float sc = pow2i(fexp[qi][sgn ? 1 : 0]);
    const uint32_t sel = (uint32_t)l | ((uint32_t)(4 + l) << 4);
    uint32_t word[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = 32 * (SP::WPL * t + g) + 8 * i + st + 4 * r;
        const float x = q < nq ? coef * (sgn ? p[(int64_t)q * D + j] : qr[(int64_t)q * D + j]) : 0.f;
        w[i] = (uint32_t)__float2int_rn(x * sc) + 0x80808080u;  // balanced limbs: byte l ^ 0x80
      }
      word[r] = __byte_perm(__byte_perm(w[0], w[1], sel), __byte_perm(w[2], w[3], sel), 0x5410) ^ 0x80808080u;
    }
    out[idx] = make_uint2(word[0], word[1]);
  }
}

// Shared-memory layout of the scan (byte offsets; the lists depend on k, the row buffers on nbuf).
struct ScanLayout {
  size_t kq, xch, rows, rowbuf, rc, rs, rn, rr, ls, li, bars, total;
  int nbuf;
};

template <int BK, int D>
__host__ __device__ inline ScanLayout scan_layout(int k, int nbuf) {
  using SP = SearchMma<BK, D>;
  auto up16 = [](size_t x) { return (x + 15) & ~(size_t)15; };
  ScanLayout L;
  L.nbuf = nbuf;
  L.kq = (size_t)SP::FRAG_WORDS * 4;
  L.xch = L.kq + kSmQ * 16;
  L.rows = L.xch + (size_t)8 * 4 * 2 * 32 * 4;  // [warp][e][code, sign][lane] f32
  L.rowbuf = (size_t)kSmRB * (SP::CODE_BYTES + SP::SIGN_BYTES + 8);
  L.rc = 0;
  L.rs = L.rc + (size_t)kSmRB * SP::CODE_BYTES;
  L.rn = L.rs + (size_t)kSmRB * SP::SIGN_BYTES;
  L.rr = L.rn + (size_t)kSmRB * 4;
  L.ls = L.rows + (size_t)nbuf * L.rowbuf;
  L.li = L.ls + up16((size_t)8 * kSmQ * k * 4);
  L.bars = L.li + up16((size_t)8 * kSmQ * k * 8);
  L.total = L.bars + 16;
  return L;
}

// Warp w scores rows [32 (w & 3), 32 (w & 3) + 32) of each 128-row block (two m-tiles) over one
// half of the k-steps of every plane (kh = w >> 2: half of a lane's words, or at d = 128 half of
// the four bit positions st), so that each query-fragment load feeds two MMAs and six independent
// accumulator chains run per warp.  The two halves swap partial sums through shared memory; warp
// (rg, kh) then finishes m-tile kh of its row group.
template <int BK, int D>
__global__ void __launch_bounds__(kSmThreads, 2)
search_mma_kernel(TqConsts c, const uint2 *__restrict__ frag, const float *__restrict__ kq, int nq, tq_packed db,
                  int64_t n, int k, int64_t rows_per_shard, int shards, int nbuf, float *__restrict__ cand_s,
                  int64_t *__restrict__ cand_i) {
  using SP = SearchMma<BK, D>;
  constexpr int WPL = SP::WPL;
  constexpr int HW = WPL >= 2 ? WPL / 2 : 1;  // words per row and plane this warp loads
  constexpr int NST = WPL >= 2 ? 4 : 2;       // bit positions st per word this warp covers
  extern __shared__ __align__(16) unsigned char smem[];
  const ScanLayout L = scan_layout<BK, D>(k, nbuf);
  const uint2 *sfrag = reinterpret_cast<const uint2 *>(smem);
  const float *skq = reinterpret_cast<const float *>(smem + L.kq);
  float *xch = reinterpret_cast<float *>(smem + L.xch);
  float *ls = reinterpret_cast<float *>(smem + L.ls);  // [warp][q][k]
  int64_t *li = reinterpret_cast<int64_t *>(smem + L.li);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  // the query tiles of a shard are adjacent in launch order (x fastest), so they run at the same
  // time and the shard's rows come from DRAM once, the other tiles reading them from L2
  const int tile = blockIdx.x, shard = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, t = lane & 3;
  const int rg = warp & 3, kh = warp >> 2;
  const int g0 = WPL >= 2 ? kh * HW : 0, st0 = WPL >= 2 ? 0 : 2 * kh;
  const int64_t r_begin = (int64_t)shard * rows_per_shard;
  const int64_t r_end = min(n, r_begin + rows_per_shard);
  const int nblk = r_end > r_begin ? (int)((r_end - r_begin + kSmRB - 1) / kSmRB) : 0;

  if (tid == 0) {
    for (int b = 0; b < nbuf; ++b) mbar_init(&bars[b], 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  for (int i = tid; i < 8 * kSmQ * k; i += kSmThreads) {
    ls[i] = -INFINITY;
    li[i] = INT64_MAX;
  }
  __syncthreads();
  // block b's rows into buffer b % nbuf, with the tile's query fragments on the first barrier
  auto issue = [&](int b) {
    if (tid != 0) return;
    const int64_t r0 = r_begin + (int64_t)b * kSmRB;
    const int nr = (int)min((int64_t)kSmRB, r_end - r0);
    unsigned char *buf = smem + L.rows + (size_t)(b % nbuf) * L.rowbuf;
    uint64_t *bar = &bars[b % nbuf];
    const int nr4 = nr & ~3;  // 16-byte multiples by bulk copy, the last few rows by plain loads
    const unsigned fb = b == 0 ? (unsigned)SP::FRAG_WORDS * 4u + kSmQ * 16u : 0u;
    mbar_expect_arrive(bar, (unsigned)nr * (SP::CODE_BYTES + SP::SIGN_BYTES) + (unsigned)nr4 * 8u + fb);
    bulk_g2s(buf + L.rc, static_cast<const char *>(db.codes) + r0 * SP::CODE_BYTES, (unsigned)nr * SP::CODE_BYTES,
             bar);
    bulk_g2s(buf + L.rs, static_cast<const char *>(db.signs) + r0 * SP::SIGN_BYTES, (unsigned)nr * SP::SIGN_BYTES,
             bar);
    if (nr4 > 0) {
      bulk_g2s(buf + L.rn, static_cast<const float *>(db.norm) + r0, (unsigned)nr4 * 4, bar);
      bulk_g2s(buf + L.rr, static_cast<const float *>(db.rnorm) + r0, (unsigned)nr4 * 4, bar);
    }
    for (int r = nr4; r < nr; ++r) {
      reinterpret_cast<float *>(buf + L.rn)[r] = static_cast<const float *>(db.norm)[r0 + r];  // fp32 norms only
      reinterpret_cast<float *>(buf + L.rr)[r] = static_cast<const float *>(db.rnorm)[r0 + r];
    }
    if (b == 0) {
      bulk_g2s(smem, frag + (int64_t)tile * (SP::FRAG_WORDS / 2), (unsigned)SP::FRAG_WORDS * 4u, bar);
      bulk_g2s(smem + L.kq, kq + (int64_t)tile * kSmQ * 4, kSmQ * 16u, bar);
    }
  };
  // multipliers moving bit st + 8 i (resp. st + 4 + 8 i) of a word to bit 7 of byte i, from a
  // runtime 1 so that they stay multiplies
  const uint32_t one = (uint32_t)(c.d / D);
  // this lane's two queries (columns 2t, 2t + 1)
  const int qa = 2 * t, qb = 2 * t + 1;
  float *wls = ls + (size_t)warp * kSmQ * k;
  int64_t *wli = li + (size_t)warp * kSmQ * k;

  if (nblk > 0) issue(0);
  bool failed = false;
  for (int b = 0; b < nblk; ++b) {
    if (nbuf == 2 && b + 1 < nblk) issue(b + 1);
    if (!__syncthreads_and(mbar_wait_bounded(&bars[b % nbuf], (unsigned)(b / nbuf) & 1u))) {
      failed = true;
      break;
    }
    const unsigned char *buf = smem + L.rows + (size_t)(b % nbuf) * L.rowbuf;
    const int64_t r0 = r_begin + (int64_t)b * kSmRB;
    // rows of m-tile mt: 32 rg + 16 mt + gid (+ 8)
    int acc[2][2][kSmL][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int l = 0; l < kSmL; ++l)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][x][l][e] = 0;
    uint32_t par[4][HW];
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
      for (int g = 0; g < HW; ++g) par[h][g] = 0u;
#pragma unroll 1
    for (int P = 0; P < SP::PL; ++P) {
      const bool sgn = P == SP::PL - 1;
      const bool parity = BK == 3 && P == 3;
      uint32_t w[4][HW];  // rows 32 rg + {gid, gid + 8, 16 + gid, 24 + gid}
      if (parity) {
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
          for (int g = 0; g < HW; ++g) w[h][g] = par[h][g];
      } else {
        const uint32_t *base = sgn ? reinterpret_cast<const uint32_t *>(buf + L.rs)
                                   : reinterpret_cast<const uint32_t *>(buf + L.rc) + P * (D / 32);
        const int stride = sgn ? D / 32 : BK * D / 32;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint32_t *src = base + (32 * rg + 8 * h + gid) * stride + WPL * t + g0;
          if constexpr (HW == 4) {
            const uint4 u = *reinterpret_cast<const uint4 *>(src);
            w[h][0] = u.x;
            w[h][1] = u.y;
            w[h][2] = u.z;
            w[h][3] = u.w;
          } else if constexpr (HW == 2) {
            const uint2 u = *reinterpret_cast<const uint2 *>(src);
            w[h][0] = u.x;
            w[h][1] = u.y;
          } else {
#pragma unroll
            for (int g = 0; g < HW; ++g) w[h][g] = src[g];
          }
        }
        if (BK == 3 && P < 3) {
#pragma unroll
          for (int h = 0; h < 4; ++h)
#pragma unroll
            for (int g = 0; g < HW; ++g) par[h][g] ^= w[h][g];
        }
      }
      const int pt = sgn ? 1 : 0;
#pragma unroll
      for (int g = 0; g < HW; ++g)
#pragma unroll
        for (int sti = 0; sti < NST; ++sti) {
          const int st = st0 + sti;
          const uint32_t m0 = one << (7 - st), m1 = one << (3 - st);
          const uint2 *f = sfrag + (((P * WPL + g0 + g) * 4 + st) * kSmL) * 32 + lane;
          uint2 fb[kSmL];
#pragma unroll
          for (int l = 0; l < kSmL; ++l) fb[l] = f[l * 32];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const uint32_t a0 = mul_lo(w[2 * mt][g], m0) & 0x80808080u;
            const uint32_t a1 = mul_lo(w[2 * mt + 1][g], m0) & 0x80808080u;
            const uint32_t a2 = mul_lo(w[2 * mt][g], m1) & 0x80808080u;
            const uint32_t a3 = mul_lo(w[2 * mt + 1][g], m1) & 0x80808080u;
#pragma unroll
            for (int l = 0; l < kSmL; ++l) {
              if (pt) mma_u8s8(acc[mt][1][l], a0, a1, a2, a3, fb[l].x, fb[l].y);
              else mma_u8s8(acc[mt][0][l], a0, a1, a2, a3, fb[l].x, fb[l].y);
            }
          }
        }
    }
    // this half's sums of both m-tiles; hand the other m-tile's to the partner warp
    float part[2][4][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int x = 0; x < 2; ++x)
          part[mt][e][x] = (float)acc[mt][x][0][e] + 256.f * (float)acc[mt][x][1][e] +
                           65536.f * (float)acc[mt][x][2][e];
    {
      float *o = xch + (size_t)warp * 256 + lane;
#pragma unroll
      for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int x = 0; x < 2; ++x) o[(e * 2 + x) * 32] = kh ? part[0][e][x] : part[1][e][x];
    }
    __syncthreads();
    const float *in = xch + (size_t)(warp ^ 4) * 256 + lane;
    // scores: e = 0 (row lo, query qa), 1 (lo, qb), 2 (hi, qa), 3 (hi, qb)
    const float *nrm = reinterpret_cast<const float *>(buf + L.rn);
    const float *rnm = reinterpret_cast<const float *>(buf + L.rr);
    const int rlo = 32 * rg + 16 * kh + gid, rhi = rlo + 8;
    float sc[4];
    int64_t ix[4];
    bool cand[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = e < 2 ? rlo : rhi, q = (e & 1) ? qb : qa;
      const float dc = (kh ? part[1][e][0] : part[0][e][0]) + in[(e * 2) * 32];
      const float ds = (kh ? part[1][e][1] : part[0][e][1]) + in[(e * 2 + 1) * 32];
      const float a = fmaf(dc, skq[4 * q], -skq[4 * q + 2]);
      const float s2 = fmaf(ds, skq[4 * q + 1], -skq[4 * q + 3]);
      sc[e] = nrm[r] * fmaf(c.qjl_scale * rnm[r], s2, a);
      ix[e] = r0 + r;
      const bool ok = r0 + r < r_end && tile * kSmQ + q < nq;
      cand[e] = ok && tq_better(sc[e], ix[e], wls[q * k + k - 1], wli[q * k + k - 1]);
    }
    // rare: candidates better than a query's current k-th best go into the warp's sorted list,
    // one lane at a time
    unsigned m = __ballot_sync(TQ_FULL_MASK, cand[0] || cand[1] || cand[2] || cand[3]);
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      if (lane == src) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = (e & 1) ? qb : qa;
          float *Ls = wls + q * k;
          int64_t *Li = wli + q * k;
          if (!cand[e] || !tq_better(sc[e], ix[e], Ls[k - 1], Li[k - 1])) continue;
          int pos = k - 1;
          while (pos > 0 && tq_better(sc[e], ix[e], Ls[pos - 1], Li[pos - 1])) {
            Ls[pos] = Ls[pos - 1];
            Li[pos] = Li[pos - 1];
            --pos;
          }
          Ls[pos] = sc[e];
          Li[pos] = ix[e];
        }
      }
      __syncwarp();
    }
    __syncthreads();  // the buffer and the exchange area are refilled next
    if (nbuf == 1 && b + 1 < nblk) issue(b + 1);
  }
  if (failed) {
    if (tid == 0) {
      atomicOr(&g_tq_device_flags, kFlagStagingTimeout);
      for (int b = 0; b < nbuf; ++b) mbar_wait_bounded(&bars[b], 0u);
      mbar_wait_bounded(&bars[0], 1u);
    }
    __syncthreads();
    return;
  }
  // warp q merges query q's 8 warp lists (8 x k candidates) and writes the shard's top-k
  const int q = tile * kSmQ + warp;
  if (q >= nq) return;
  float bs = -INFINITY;
  int64_t bi = INT64_MAX;
  for (int w2 = 0; w2 < 8; ++w2) {
    const float s = lane < k ? ls[((size_t)w2 * kSmQ + warp) * k + lane] : -INFINITY;
    const int64_t i = lane < k ? li[((size_t)w2 * kSmQ + warp) * k + lane] : INT64_MAX;
    warp_topk_insert(bs, bi, k, s, i, lane < k && i != INT64_MAX);
  }
  if (lane < k) {
    const int64_t o = ((int64_t)q * shards + shard) * k + lane;
    cand_s[o] = bs;
    cand_i[o] = bi;
  }
}

// Per-SM shared memory for resident CTAs (228 KB, 1 KB of it reserved per CTA) and the largest
// per-CTA allocation (227 KB).
constexpr size_t kSmemPerSm = 233472, kSmemPerCta = 232448, kSmemReserved = 1024;

// Buffer count and resident CTAs per SM: two CTAs (one buffer each, or two if they fit) when two
// fit, else one CTA with two buffers when they fit.
template <int BK, int D>
ScanLayout scan_config(int k, int *ctas_per_sm) {
  ScanLayout two = scan_layout<BK, D>(k, 2), one = scan_layout<BK, D>(k, 1);
  if (2 * (two.total + kSmemReserved) <= kSmemPerSm) { *ctas_per_sm = 2; return two; }
  if (2 * (one.total + kSmemReserved) <= kSmemPerSm) { *ctas_per_sm = 2; return one; }
  *ctas_per_sm = 1;
  return two.total <= kSmemPerCta ? two : one;
}

template <int BK, int D>
int pick_shards(int nq, int64_t n, int k) {
  int per_sm = 1;
  scan_config<BK, D>(k, &per_sm);
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) ==
                                                  cudaSuccess && v > 0)
      sms = v;
    else
      sms = 148;
  }
  // cost = waves x (blocks per shard + about two blocks of per-CTA start-up and final merge);
  // shards of at least four blocks
  const int64_t tiles = (nq + kSmQ - 1) / kSmQ, slots = (int64_t)sms * per_sm;
  const int64_t nb = (n + kSmRB - 1) / kSmRB;
  const int64_t max_s = std::max<int64_t>(1, std::min<int64_t>(4096, nb / 4));
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

template <int BK, int D>
cudaError_t launch_mma_search(const TqConsts &c, int shards, const float *qr, const float *p, int nq,
                              const tq_packed &db, int64_t n, int k, void *fragws, float *cand_s,
                              int64_t *cand_i, cudaStream_t st) {
  using SP = SearchMma<BK, D>;
  const int tiles = (nq + kSmQ - 1) / kSmQ;
  uint2 *frag = static_cast<uint2 *>(fragws);
  float *kq = reinterpret_cast<float *>(static_cast<char *>(fragws) +
                                        tq_align_up((int64_t)tiles * SP::FRAG_WORDS * 4, 256));
  int per_sm = 1;
  const ScanLayout L = scan_config<BK, D>(k, &per_sm);
  tq_prof_begin(TQK_SEARCH_SCAN, st);
  search_frag_kernel<BK, D><<<tiles, kSmThreads, 0, st>>>(c, qr, p, nq, frag, kq);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    e = tq_smem_limit(reinterpret_cast<const void *>(search_mma_kernel<BK, D>), (int)L.total);
    if (e == cudaSuccess) {
      const int64_t rows_per_shard = ((n + shards - 1) / shards + kSmRB - 1) / kSmRB * kSmRB;
      search_mma_kernel<BK, D><<<dim3((unsigned)tiles, (unsigned)shards), kSmThreads, L.total, st>>>(
          c, frag, kq, nq, db, n, k, rows_per_shard, shards, L.nbuf, cand_s, cand_i);
      e = cudaGetLastError();
    }
  }
  tq_prof_end(TQK_SEARCH_SCAN, st);
  return e;
}

}  // namespace

bool search_mma_eligible(const TqConsts &c) {
  return (c.d == 128 || c.d == 256 || c.d == 512 || c.d == 1024) && c.m == c.d && c.bits >= 1 && c.bits <= 3 &&
         c.fast_ok && c.layout == TQ_LAYOUT_ROWS;
}

size_t search_mma_frag_bytes(const TqConsts &c, int nq) {
  const int tiles = (nq + kSmQ - 1) / kSmQ;
  const int pl = c.bits + (c.bits == 3 ? 1 : 0) + 1;
  const int64_t words = (int64_t)pl * (c.d / 128) * 4 * kSmL * 32 * 2;
  return (size_t)tq_align_up((int64_t)tiles * words * 4, 256) + (size_t)tq_align_up((int64_t)tiles * kSmQ * 16, 256);
}

int search_mma_shards(const TqConsts &c, int nq, int64_t n, int k) {
#define TQ_SM(BKV, DV) \
  if (c.bits == BKV && c.d == DV) return pick_shards<BKV, DV>(nq, n, k);
  TQ_SM(1, 128) TQ_SM(2, 128) TQ_SM(3, 128)
  TQ_SM(1, 256) TQ_SM(2, 256) TQ_SM(3, 256)
  TQ_SM(1, 512) TQ_SM(2, 512) TQ_SM(3, 512)
  TQ_SM(1, 1024) TQ_SM(2, 1024) TQ_SM(3, 1024)
#undef TQ_SM
  return 1;
}

cudaError_t launch_search_mma(const TqConsts &c, int shards, const float *qr, const float *p, int nq,
                              const tq_packed &db, int64_t n, int k, void *fragws, float *cand_s, int64_t *cand_i,
                              cudaStream_t st) {
#define TQ_SM(BKV, DV)                 \
  if (c.bits == BKV && c.d == DV)      \
    return launch_mma_search<BKV, DV>(c, shards, qr, p, nq, db, n, k, fragws, cand_s, cand_i, st);
  TQ_SM(1, 128) TQ_SM(2, 128) TQ_SM(3, 128)
  TQ_SM(1, 256) TQ_SM(2, 256) TQ_SM(3, 256)
  TQ_SM(1, 512) TQ_SM(2, 512) TQ_SM(3, 512)
  TQ_SM(1, 1024) TQ_SM(2, 1024) TQ_SM(3, 1024)
#undef TQ_SM
  return cudaErrorInvalidValue;
}

// The device flags of this translation unit's kernels (see tq_device_status).
TQ_DEVICE_FLAGS_ACCESSOR(search_mma_device_flags)
