// Decode attention over the compressed KV cache, split over the context (one CTA per
// (split, KV head, sequence)) and then combined.
//
// Per CTA, for tiles of 128 tokens (one thread per token):
//   logits  l_t = scale * nu_t (<q', c_K[code_t]> + sqrt(pi/2)/m gamma_t <2 bits_t - 1, p>)
//           (PolarQuant keys: <q', y^_t>, y^_t the direction rebuilt from the angle codes)
//           for the G query heads that share the KV head ("谷歌 TurboQuant 深度拆解" 第二部分
//           第二步 and 第三部分 "推理速度": logits against the compressed keys);
//   online softmax: running max and sum per head, earlier partial sums rescaled;
//   values  accumulated in the ROTATED domain: o~_j += w_t nu_t c_V[codeV_t,j], one thread per
//           coordinate j (all threads read the same token's packed words: broadcast loads).
// The combine kernel merges the splits with their log-sum-exp weights and applies the inverse
// rotation once per output: o = D_V (1/sqrt d) H o~ / L.  Because the rotation is linear and
// orthogonal, this equals the weighted sum of the individually reconstructed value vectors.
#include <cmath>

#include "device_common.cuh"
#include "polar_device.cuh"

namespace {

constexpr int kAtThreads = 128;
constexpr int kAtTile = 128;
constexpr int kAtWarps = kAtThreads / 32;
constexpr int kMaxDpt = 1024 / kAtThreads;  // coordinates per thread in the value sum

struct AttnArgs {
  int batch, hq, hkv, max_len, chunk, splits, block_size, max_blocks;
  int64_t ctx_stride;
  float scale;
  const int32_t *seq_lens;
  const int32_t *block_table;
  tq_packed k, v;
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) x = fmaxf(x, __shfl_xor_sync(TQ_FULL_MASK, x, s));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) x += __shfl_xor_sync(TQ_FULL_MASK, x, s);
  return x;
}

// KP / VP: PolarQuant keys / values (d = 128): the key scores through the reconstructed direction,
// a value coordinate as the product of cos / sin of the angles along its path.
template <int G, bool KP, bool VP>
__global__ void __launch_bounds__(kAtThreads)
attend_split_kernel(TqConsts kc, TqConsts vc, AttnArgs a, const float *__restrict__ qr,
                    const float *__restrict__ p, float *__restrict__ part) {
  __shared__ PolarTab ktab, vtab;
  extern __shared__ float sm[];
  const int d = kc.d, m = kc.m;
  float *qs = sm;                        // [d][G]
  float *ps = qs + d * G;                // [m][G]
  float *lg = ps + m * G;                // [G][tile] weights * value norms
  float *red = lg + G * kAtTile;         // [G][warps] tile maxima
  float *red2 = red + G * kAtWarps;      // [G][warps] tile sums
  float *centK = red2 + G * kAtWarps;    // [16]
  float *centV = centK + 16;             // [16]
  int64_t *sl = reinterpret_cast<int64_t *>(centV + 16);  // [tile] slots (-1 = masked)

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int L = a.seq_lens[b];
  L = L < 0 ? 0 : (L > a.max_len ? a.max_len : L);
  const int t0 = s * a.chunk;
  const int t1 = min(L, t0 + a.chunk);

  const int64_t qbase = (int64_t)b * a.hq + (int64_t)h * G;
  for (int i = tid; i < d * G; i += kAtThreads) qs[i] = qr[(qbase + i % G) * d + i / G];
  for (int i = tid; i < m * G; i += kAtThreads) ps[i] = p[(qbase + i % G) * m + i / G];
  if (tid < TQ_MAX_LEVELS) {
    centK[tid] = kc.centroids[tid];
    centV[tid] = vc.centroids[tid];
  }
  if (KP) polar_tab_stage(ktab, kc.polar_tab, tid, kAtThreads);
  if (VP) polar_tab_stage(vtab, vc.polar_tab, tid, kAtThreads);
  __syncthreads();

  const uint32_t *kcodes = static_cast<const uint32_t *>(a.k.codes);
  const uint32_t *ksigns = static_cast<const uint32_t *>(a.k.signs);
  const uint32_t *vcodes = static_cast<const uint32_t *>(a.v.codes);

  float mrun[G], lrun[G], acc[G][kMaxDpt];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    mrun[g] = -INFINITY;
    lrun[g] = 0.f;
#pragma unroll
    for (int dd = 0; dd < kMaxDpt; ++dd) acc[g][dd] = 0.f;
  }

  for (int tt = t0; tt < t1; tt += kAtTile) {
    const int t = tt + tid;
    bool ok = t < t1;
    int64_t slot = -1;
    if (ok) {
      if (a.block_table) {
        const int blk = a.block_table[(int64_t)b * a.max_blocks + t / a.block_size];
        slot = blk < 0 ? -1 : ((int64_t)blk * a.hkv + h) * a.block_size + t % a.block_size;
      } else {
        slot = ((int64_t)b * a.hkv + h) * a.ctx_stride + t;
      }
      ok = slot >= 0 && slot < a.k.capacity && slot < a.v.capacity;
    }
    float sc[G];
    float nuv = 0.f;
    if (ok) {
      const uint32_t *kr = kcodes + slot * kc.code_words, *ks = m > 0 ? ksigns + slot * kc.sign_words : nullptr;
      const float nuk = ld_norm(a.k.norm, slot, kc.norm16), gk = m > 0 ? ld_norm(a.k.rnorm, slot, kc.norm16) : 0.f;
      if constexpr (KP)
        polar_scores<G>(kc, kr, ks, nuk, gk, qs, ps, ktab, sc);
      else
        estimate_scores<G>(kc, kr, ks, nuk, gk, qs, ps, centK, sc);
#pragma unroll
      for (int g = 0; g < G; ++g) sc[g] *= a.scale;
      nuv = ld_norm(a.v.norm, slot, vc.norm16);
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) sc[g] = -INFINITY;
    }
    sl[tid] = ok ? slot : -1;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mx = warp_max(sc[g]);
      if (lane == 0) red[g * kAtWarps + warp] = mx;
    }
    __syncthreads();
    float mnew[G], alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float tm = red[g * kAtWarps];
#pragma unroll
      for (int w = 1; w < kAtWarps; ++w) tm = fmaxf(tm, red[g * kAtWarps + w]);
      mnew[g] = fmaxf(mrun[g], tm);
      alpha[g] = (mrun[g] == -INFINITY) ? 0.f : __expf(mrun[g] - mnew[g]);
      const float w = ok ? __expf(sc[g] - mnew[g]) : 0.f;
      lg[g * kAtTile + tid] = w * nuv;
      const float ws = warp_sum(w);
      if (lane == 0) red2[g * kAtWarps + warp] = ws;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float ts = 0.f;
#pragma unroll
      for (int w = 0; w < kAtWarps; ++w) ts += red2[g * kAtWarps + w];
      lrun[g] = lrun[g] * alpha[g] + ts;
      mrun[g] = mnew[g];
#pragma unroll
      for (int dd = 0; dd < kMaxDpt; ++dd) acc[g][dd] *= alpha[g];
    }
    const int nt = min(kAtTile, t1 - tt);
    for (int i = 0; i < nt; ++i) {
      const int64_t si = sl[i];
      if (si < 0) continue;
      float wv[G];
#pragma unroll
      for (int g = 0; g < G; ++g) wv[g] = lg[g * kAtTile + i];
#pragma unroll
      for (int dd = 0; dd < kMaxDpt; ++dd) {
        const int j = tid + dd * kAtThreads;
        if (j < d) {
          float cv;
          if constexpr (VP)
            cv = polar_coord(vcodes + si * vc.code_words, j, vc.bits, vtab);
          else
            cv = centV[slot_code(vcodes, si, j, vc)];
#pragma unroll
          for (int g = 0; g < G; ++g) acc[g][dd] = fmaf(wv[g], cv, acc[g][dd]);
        }
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int64_t base = (((int64_t)b * a.hq + (int64_t)h * G + g) * a.splits + s) * (d + 4);
    if (tid == 0) {
      part[base] = mrun[g];
      part[base + 1] = lrun[g];
    }
#pragma unroll
    for (int dd = 0; dd < kMaxDpt; ++dd) {
      const int j = tid + dd * kAtThreads;
      if (j < d) part[base + 2 + j] = acc[g][dd];
    }
  }
}

constexpr int kCbThreads = 512;

__device__ __forceinline__ float block_reduce(float v, float *red, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const float o = __shfl_xor_sync(TQ_FULL_MASK, v, s);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < nw; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

// Merge the split partials of one (sequence, query head) with their log-sum-exp weights, then
// undo the rotation once: o = D_V (1/sqrt d) H (sum_s e^{m_s - M} o~_s) / (sum_s e^{m_s - M} l_s).
// 512 threads: the splits are summed in parallel by (coordinate, split group) pairs.
__global__ void __launch_bounds__(kCbThreads)
attend_combine_kernel(TqConsts vc, int splits, const float *__restrict__ part, float *__restrict__ out) {
  extern __shared__ float sm[];
  const int d = vc.d;
  const int ngroups = kCbThreads >= d ? kCbThreads / d : 1;
  float *f = sm;                       // [splits]
  float *y = f + splits;               // [d]
  float *acc = y + d;                  // [ngroups][d]
  float *red = acc + ngroups * d;      // [32]
  const int64_t bh = blockIdx.x;
  const float *pb = part + bh * splits * (d + 4);
  float m = -INFINITY;
  for (int s = threadIdx.x; s < splits; s += blockDim.x) m = fmaxf(m, pb[(int64_t)s * (d + 4)]);
  const float M = block_reduce(m, red, true);
  float l = 0.f;
  for (int s = threadIdx.x; s < splits; s += blockDim.x) {
    const float ms = pb[(int64_t)s * (d + 4)];
    const float fs = (ms == -INFINITY) ? 0.f : __expf(ms - M);
    f[s] = fs;
    l += pb[(int64_t)s * (d + 4) + 1] * fs;
  }
  const float L = block_reduce(l, red, false);  // its barriers also publish f[]
  for (int idx = threadIdx.x; idx < ngroups * d; idx += blockDim.x) {
    const int j = idx % d, g = idx / d;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int s = g;
    for (; s + 3 * ngroups < splits; s += 4 * ngroups) {  // four independent loads in flight
      const float v0 = pb[(int64_t)s * (d + 4) + 2 + j];
      const float v1 = pb[(int64_t)(s + ngroups) * (d + 4) + 2 + j];
      const float v2 = pb[(int64_t)(s + 2 * ngroups) * (d + 4) + 2 + j];
      const float v3 = pb[(int64_t)(s + 3 * ngroups) * (d + 4) + 2 + j];
      a0 = fmaf(v0, f[s], a0);
      a1 = fmaf(v1, f[s + ngroups], a1);
      a2 = fmaf(v2, f[s + 2 * ngroups], a2);
      a3 = fmaf(v3, f[s + 3 * ngroups], a3);
    }
    for (; s < splits; s += ngroups) a0 = fmaf(pb[(int64_t)s * (d + 4) + 2 + j], f[s], a0);
    acc[g * d + j] = (a0 + a1) + (a2 + a3);
  }
  __syncthreads();
  const float inv = L > 0.f ? 1.f / L : 0.f;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float a = 0.f;
    for (int g = 0; g < ngroups; ++g) a += acc[g * d + j];
    y[j] = a * inv;
  }
  __syncthreads();
  for (int hh = 1; hh < d; hh <<= 1) {
    for (int i = threadIdx.x; i < d / 2; i += blockDim.x) {
      const int lo = (i / hh) * 2 * hh + (i % hh);
      const float a0 = y[lo], b0 = y[lo + hh];
      y[lo] = a0 + b0;
      y[lo + hh] = a0 - b0;
    }
    __syncthreads();
  }
  for (int j = threadIdx.x; j < d; j += blockDim.x) out[bh * d + j] = vc.signs[j] * y[j] * vc.inv_sqrt_d;
}

template <int G>
cudaError_t launch_split(const TqConsts &kc, const TqConsts &vc, const AttnArgs &a, dim3 grid,
                         const float *qr, const float *p, float *part, cudaStream_t st) {
  const size_t smem = sizeof(float) * ((size_t)(kc.d + kc.m) * G + (size_t)G * kAtTile +
                                       2 * G * kAtWarps + 32) +
                      sizeof(int64_t) * kAtTile;
  auto kern = kc.polar ? (vc.polar ? attend_split_kernel<G, true, true> : attend_split_kernel<G, true, false>)
                       : (vc.polar ? attend_split_kernel<G, false, true> : attend_split_kernel<G, false, false>);
  cudaError_t e = tq_smem_limit(reinterpret_cast<const void *>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  tq_prof_begin(TQK_ATTEND_SPLIT, st);
  kern<<<grid, kAtThreads, smem, st>>>(kc, vc, a, qr, p, part);
  tq_prof_end(TQK_ATTEND_SPLIT, st);
  return cudaGetLastError();
}

}  // namespace

AttnPlan attn_plan(const tq_attn_desc &desc, const TqConsts &kc, const TqConsts &vc) {
  AttnPlan p;
  p.group = desc.n_q_heads / desc.n_kv_heads;
  p.fast = attn_fast_eligible(kc, vc, desc);
  p.fused = false;
  p.extra = 0;
  if (p.fast) {
    const int maxlen = desc.max_seq_len > 0 ? desc.max_seq_len : 1;
    p.chunk = attn_fast_chunk(desc);
    p.splits = (maxlen + p.chunk - 1) / p.chunk;
    p.fused = p.splits <= kFusedMaxSplits;
    p.extra = attn_fast_extra_bytes(kc, desc);
    return p;
  }
  const int64_t rows = (int64_t)desc.batch * desc.n_kv_heads;
  const int maxlen = desc.max_seq_len > 0 ? desc.max_seq_len : 1;
  const int64_t want = rows > 0 ? (4 * 148 + rows - 1) / rows : 1;
  int64_t chunk = ((int64_t)maxlen + want - 1) / want;
  chunk = (chunk + kAtTile - 1) / kAtTile * kAtTile;
  if (chunk < 512) chunk = 512;
  p.chunk = (int)chunk;
  p.splits = (int)((maxlen + chunk - 1) / chunk);
  return p;
}

size_t attn_partials_bytes(const tq_attn_desc &desc, const AttnPlan &plan, int d) {
  return (size_t)tq_align_up((int64_t)sizeof(float) * desc.batch * desc.n_q_heads * plan.splits * (d + 4), 256) +
         plan.extra;
}

cudaError_t launch_attend(const TqConsts &kc, const TqConsts &vc, const tq_attn_desc &desc,
                          const AttnPlan &plan, const void *q, int dtype, const float *qr, const float *p,
                          float *partials, float *out, cudaStream_t st) {
  if (desc.batch <= 0) return cudaSuccess;
  AttnArgs a;
  a.batch = desc.batch;
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
  dim3 grid((unsigned)plan.splits, (unsigned)desc.n_kv_heads, (unsigned)desc.batch);
  cudaError_t e;
  if (plan.fast) {
    void *extra = reinterpret_cast<char *>(partials) +
                  tq_align_up((int64_t)sizeof(float) * desc.batch * desc.n_q_heads * plan.splits * (kc.d + 4), 256);
    e = launch_attend_fast(kc, vc, desc, plan, q, dtype, extra, partials, plan.fused ? out : nullptr, st);
    if (e != cudaSuccess || plan.fused) return e;
  } else switch (plan.group) {
    case 1: e = launch_split<1>(kc, vc, a, grid, qr, p, partials, st); break;
    case 2: e = launch_split<2>(kc, vc, a, grid, qr, p, partials, st); break;
    case 4: e = launch_split<4>(kc, vc, a, grid, qr, p, partials, st); break;
    case 8: e = launch_split<8>(kc, vc, a, grid, qr, p, partials, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_attend_combine(vc, desc, plan, partials, out, st);
}

cudaError_t launch_attend_combine(const TqConsts &vc, const tq_attn_desc &desc, const AttnPlan &plan,
                                  const float *partials, float *out, cudaStream_t st) {
  const int ngroups = kCbThreads >= vc.d ? kCbThreads / vc.d : 1;
  const size_t smem = sizeof(float) * ((size_t)plan.splits + vc.d + (size_t)ngroups * vc.d + 32);
  cudaError_t e2 = tq_smem_limit(reinterpret_cast<const void *>(attend_combine_kernel), (int)smem);
  if (e2 != cudaSuccess) return e2;
  tq_prof_begin(TQK_ATTEND_COMBINE, st);
  attend_combine_kernel<<<(unsigned)((int64_t)desc.batch * desc.n_q_heads), kCbThreads, smem, st>>>(
      vc, plan.splits, partials, out);
  tq_prof_end(TQK_ATTEND_COMBINE, st);
  return cudaGetLastError();
}
