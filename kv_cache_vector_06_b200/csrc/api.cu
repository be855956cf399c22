// C-ABI entry points of libtq: argument validation, context management and orchestration of the
// kernels.  Every data call validates on the host first and only then enqueues work on the
// caller's stream; nothing here allocates on a data call.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "tq_internal.h"

namespace {
thread_local char g_err[512] = "";

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tq_status check_spec(const tq_spec *s) {
  if (!s) return tq_fail(TQ_EINVAL, "spec is NULL");
  if (!is_pow2(s->d) || s->d < 8 || s->d > 1024)
    return tq_fail(TQ_EUNSUPPORTED, "d=%d: must be a power of two in [8, 1024]", s->d);
  if (s->mse_bits < 1 || s->mse_bits > 4)
    return tq_fail(TQ_EUNSUPPORTED, "mse_bits=%d: must be in [1, 4]", s->mse_bits);
  if (s->qjl_m < 0 || s->qjl_m > 1024 || (s->qjl_m % 32) != 0)
    return tq_fail(TQ_EUNSUPPORTED, "qjl_m=%d: must be 0 or a multiple of 32 in [32, 1024]",
                   s->qjl_m);
  if (s->layout != TQ_LAYOUT_ROWS && s->layout != TQ_LAYOUT_BLOCK16)
    return tq_fail(TQ_EINVAL, "layout=%d: unknown", s->layout);
  if (s->layout == TQ_LAYOUT_BLOCK16 && s->qjl_m != 0)
    return tq_fail(TQ_EUNSUPPORTED, "TQ_LAYOUT_BLOCK16 holds MSE-only codes (qjl_m must be 0)");
  if (s->norm_bits != 0 && s->norm_bits != 16 && s->norm_bits != 32)
    return tq_fail(TQ_EINVAL, "norm_bits=%d: must be 32 (or 0) or 16", s->norm_bits);
  return TQ_OK;
}

// Address of stored norm i (fp16 or fp32 per the context).
void *norm_at(const tq_ctx *c, void *p, int64_t i) { return static_cast<char *>(p) + i * (c->k.norm16 ? 2 : 4); }

tq_status check_ctx(const tq_ctx *c, const char *name) {
  if (!c) return tq_fail(TQ_EINVAL, "%s is NULL", name);
  return TQ_OK;
}


tq_status check_packed(const tq_ctx *c, const tq_packed &p, int64_t need, const char *name,
                       bool need_signs) {
  if (!p.codes || !p.norm) return tq_fail(TQ_EINVAL, "%s: codes/norm is NULL", name);
  if (!aligned16(p.codes)) return tq_fail(TQ_EINVAL, "%s: codes not 16-byte aligned", name);
  const uintptr_t nal = c->k.norm16 ? 1u : 3u;  // fp16 or fp32 norms
  if ((reinterpret_cast<uintptr_t>(p.norm) & nal) != 0)
    return tq_fail(TQ_EINVAL, "%s: norm not %d-byte aligned", name, (int)nal + 1);
  if (need_signs && c->spec.qjl_m > 0) {
    if (!p.signs || !p.rnorm) return tq_fail(TQ_EINVAL, "%s: signs/rnorm is NULL", name);
    if (!aligned16(p.signs)) return tq_fail(TQ_EINVAL, "%s: signs not 16-byte aligned", name);
    if ((reinterpret_cast<uintptr_t>(p.rnorm) & nal) != 0)
      return tq_fail(TQ_EINVAL, "%s: rnorm not %d-byte aligned", name, (int)nal + 1);
  }
  if (p.capacity < 0) return tq_fail(TQ_EINVAL, "%s: negative capacity", name);
  if (c->spec.layout == TQ_LAYOUT_BLOCK16 && (p.capacity % 16) != 0)
    return tq_fail(TQ_EINVAL, "%s: TQ_LAYOUT_BLOCK16 needs a capacity that is a multiple of 16", name);
  if (need > p.capacity)
    return tq_fail(TQ_EINVAL, "%s: %lld slots needed, capacity %lld", name, (long long)need,
                   (long long)p.capacity);
  return TQ_OK;
}

size_t query_prep_bytes(const tq_ctx *c, int64_t nq) {
  return (size_t)tq_align_up(nq * c->spec.d * 4, 256) + (size_t)tq_align_up(nq * c->spec.qjl_m * 4, 256);
}

// q (any dtype) -> q' [nq][d] and p [nq][m] in the workspace
tq_status prep_queries(const tq_ctx *c, const void *q, tq_dtype dt, int64_t nq, float *qr, float *p,
                       cudaStream_t st) {
  cudaError_t e = launch_rotate(c->k, ROT_QUERY, q, dt, nq, c->spec.d, nullptr, 0, nullptr,
                                nullptr, nullptr, qr, st, nullptr);
  if (e != cudaSuccess) return tq_cuda_check(e, "query rotation launch");
  if (c->spec.qjl_m > 0) {
    e = launch_project(c->k, PROJ_DENSE, qr, nq, nullptr, 0, nullptr, p, st);
    if (e != cudaSuccess) return tq_cuda_check(e, "query projection launch");
  }
  return TQ_OK;
}

constexpr int64_t kEncodeChunk = 1 << 16;  // rows per residual-workspace pass
}  // namespace

tq_status tq_fail(tq_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

tq_status tq_cuda_check(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return TQ_OK;
  return tq_fail(TQ_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

extern "C" {

const char *tq_last_error(void) { return g_err; }
// The revision tags of the tensor-core kernels name the device code that a recorded profile (DRAM
// traffic per launch) was taken on; each changes whenever its kernel's code changes.
const char *tq_version(void) { return "libtq 0.4 (sm_100a; attend_mma r14; search_tc r3; encode_tc r3)"; }

tq_status tq_make_codebook(int32_t d, int32_t bits, double *centroids, double *thresholds,
                           double *mse_per_coord) {
  g_err[0] = 0;
  if (!centroids || !thresholds) return tq_fail(TQ_EINVAL, "centroids/thresholds is NULL");
  tq_spec s{d, bits, 0, TQ_LAYOUT_ROWS};
  tq_status st = check_spec(&s);
  if (st != TQ_OK) return st;
  return tq_codebook_fp64(d, bits, centroids, thresholds, mse_per_coord);
}

// Shared by tq_ctx_create (caller-drawn S) and tq_ctx_create_srht (S = P H D2 built here).
static tq_status ctx_create(const tq_spec *spec, const int8_t *rot_signs, const float *qjl_matrix,
                            const int8_t *qjl_signs, bool polar, int32_t device, tq_ctx **out) {
  if (!out) return tq_fail(TQ_EINVAL, "out is NULL");
  *out = nullptr;
  tq_status st = check_spec(spec);
  if (st != TQ_OK) return st;
  if (!rot_signs) return tq_fail(TQ_EINVAL, "rot_signs is NULL");
  if (spec->qjl_m > 0 && !qjl_matrix) return tq_fail(TQ_EINVAL, "qjl_matrix is NULL with qjl_m > 0");
  const int d = spec->d, m = spec->qjl_m, L = 1 << spec->mse_bits;
  for (int j = 0; j < d; ++j)
    if (rot_signs[j] != 1 && rot_signs[j] != -1)
      return tq_fail(TQ_EINVAL, "rot_signs[%d] = %d: must be +1 or -1", j, (int)rot_signs[j]);

  tq_ctx *c = new (std::nothrow) tq_ctx();
  if (!c) return tq_fail(TQ_ENOMEM, "host allocation failed");
  c->device = device;
  c->spec = *spec;
  c->code_bytes = tq_align_up(((int64_t)spec->mse_bits * d + 7) / 8, 16);
  c->sign_bytes = m > 0 ? tq_align_up((m + 7) / 8, 16) : 0;
  tq_codebook_fp64(d, spec->mse_bits, c->centroids, c->thresholds, &c->mse_per_coord);

  DeviceScope dev_scope;
  st = dev_scope.enter(device);
  if (st != TQ_OK) {
    delete c;
    return st;
  }
  cudaError_t e = cudaSuccess;
  float hs[1024];
  for (int j = 0; j < d; ++j) hs[j] = (float)rot_signs[j];
  float hs2[1024];
  if (qjl_signs)
    for (int j = 0; j < d; ++j) hs2[j] = (float)qjl_signs[j];
  e = cudaMalloc(&c->dev_signs, sizeof(float) * d);
  if (e == cudaSuccess && m > 0) e = cudaMalloc(&c->dev_S, sizeof(float) * (size_t)m * d);
  if (e == cudaSuccess && m > 0) e = cudaMalloc(&c->dev_St, sizeof(float) * (size_t)m * d);
  if (e == cudaSuccess && qjl_signs) e = cudaMalloc(&c->dev_qjl_signs, sizeof(float) * d);
  if (e != cudaSuccess) {
    cudaFree(c->dev_signs);
    cudaFree(c->dev_S);
    cudaFree(c->dev_St);
    delete c;
    cudaGetLastError();
    return tq_fail(TQ_ENOMEM, "cudaMalloc of context constants failed");
  }
  e = cudaMemcpy(c->dev_signs, hs, sizeof(float) * d, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && m > 0)
    e = cudaMemcpy(c->dev_S, qjl_matrix, sizeof(float) * (size_t)m * d, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && m > 0) {
    std::vector<float> st((size_t)m * d);
    for (int i = 0; i < m; ++i)
      for (int j = 0; j < d; ++j) st[(size_t)j * m + i] = qjl_matrix[(size_t)i * d + j];
    e = cudaMemcpy(c->dev_St, st.data(), sizeof(float) * (size_t)m * d, cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess && qjl_signs)
    e = cudaMemcpy(c->dev_qjl_signs, hs2, sizeof(float) * d, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && polar) {
    // PolarQuant angle tables: per level, the thresholds and the cos / sin of the centroids
    constexpr int kLv = 7;
    float tab[kLv][3][16] = {};
    for (int l = 1; l <= kLv; ++l) {
      double cc[16], tt[16];
      tq_polar_codebook_fp64(l, spec->mse_bits, cc, tt);
      for (int i = 0; i < L; ++i) {
        tab[l - 1][0][i] = i < L - 1 ? (float)tt[i] : INFINITY;
        tab[l - 1][1][i] = (float)std::cos(cc[i]);
        tab[l - 1][2][i] = (float)std::sin(cc[i]);
      }
    }
    e = cudaMalloc(&c->dev_polar, sizeof(tab));
    if (e == cudaSuccess) e = cudaMemcpy(c->dev_polar, tab, sizeof(tab), cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    cudaFree(c->dev_signs);
    cudaFree(c->dev_S);
    cudaFree(c->dev_St);
    cudaFree(c->dev_qjl_signs);
    cudaFree(c->dev_polar);
    delete c;
    return tq_cuda_check(e, "upload of context constants");
  }
  TqConsts &k = c->k;
  k.d = d;
  k.bits = spec->mse_bits;
  k.levels = L;
  k.m = m;
  k.code_words = (int)(c->code_bytes / 4);
  k.sign_words = (int)(c->sign_bytes / 4);
  k.layout = spec->layout;
  k.norm16 = spec->norm_bits == 16 ? 1 : 0;
  k.inv_sqrt_d = (float)(1.0 / std::sqrt((double)d));
  k.qjl_scale = m > 0 ? (float)(std::sqrt(M_PI / 2.0) / m) : 0.0f;
  for (int i = 0; i < TQ_MAX_LEVELS; ++i) {
    k.centroids[i] = i < L ? (float)c->centroids[i] : 0.0f;
    k.thresholds[i] = i < L - 1 ? (float)c->thresholds[i] : INFINITY;
  }
  k.signs = c->dev_signs;
  k.S = c->dev_S;
  k.St = c->dev_St;
  k.srht = qjl_signs ? 1 : 0;
  k.qjl_signs = c->dev_qjl_signs;
  k.polar = polar ? 1 : 0;
  k.polar_tab = c->dev_polar;
  // odd bit-plane expansion of the codebook for the tensor-core attention path:
  // e_S = 2^-b sum_code c[code] prod_{P in S} s_P(code), S in {0}, {1}, {2}, {0,1,2}
  k.fast_ok = 0;
  for (int i = 0; i < 4; ++i) k.plane_coef[i] = 0.f;
  k.plane_coef_sum = 0.f;
  k.plane_coef_max = 0.f;
  if (spec->mse_bits <= 3) {
    const int b = spec->mse_bits;
    const int nsets = b == 3 ? 4 : b;
    double coef[4] = {0, 0, 0, 0};
    for (int code = 0; code < L; ++code) {
      double sg[3];
      for (int P = 0; P < 3; ++P) sg[P] = ((code >> P) & 1) ? 1.0 : -1.0;
      for (int S = 0; S < nsets; ++S) {
        const double prod = S < 3 ? sg[S] : sg[0] * sg[1] * sg[2];
        coef[S] += c->centroids[code] * prod / L;
      }
    }
    double worst = 0.0;
    for (int code = 0; code < L; ++code) {
      double sg[3], rec = 0.0;
      for (int P = 0; P < 3; ++P) sg[P] = ((code >> P) & 1) ? 1.0 : -1.0;
      for (int S = 0; S < nsets; ++S) rec += coef[S] * (S < 3 ? sg[S] : sg[0] * sg[1] * sg[2]);
      worst = std::fmax(worst, std::fabs(rec - c->centroids[code]));
    }
    double sum = 0.0;
    for (int S = 0; S < nsets; ++S) {
      k.plane_coef[S] = (float)coef[S];
      k.plane_coef_max = std::fmax(k.plane_coef_max, (float)coef[S]);
      sum += coef[S];
    }
    k.plane_coef_sum = (float)sum;
    k.fast_ok = worst <= 1e-9 * std::fabs(c->centroids[L - 1]) ? 1 : 0;
  }
  if (polar) k.fast_ok = 0;  // angle codes: the bit-plane tensor-core paths do not apply
  *out = c;
  return TQ_OK;
}


tq_status tq_ctx_create(const tq_spec *spec, const int8_t *rot_signs, const float *qjl_matrix,
                        int32_t device, tq_ctx **out) {
  g_err[0] = 0;
  return ctx_create(spec, rot_signs, qjl_matrix, nullptr, false, device, out);
}

tq_status tq_ctx_create_polar(const tq_spec *spec, const int8_t *rot_signs, const float *qjl_matrix,
                              int32_t device, tq_ctx **out) {
  g_err[0] = 0;
  tq_status st = check_spec(spec);
  if (st != TQ_OK) return st;
  if (spec->d != 128 || spec->layout != TQ_LAYOUT_ROWS)
    return tq_fail(TQ_EUNSUPPORTED, "PolarQuant contexts: d = 128 and TQ_LAYOUT_ROWS");
  return ctx_create(spec, rot_signs, qjl_matrix, nullptr, true, device, out);
}

tq_status tq_polar_codebook(int32_t level, int32_t bits, double *centroids, double *thresholds) {
  g_err[0] = 0;
  if (!centroids || !thresholds) return tq_fail(TQ_EINVAL, "centroids/thresholds is NULL");
  if (level < 1 || level > 10 || bits < 1 || bits > 4)
    return tq_fail(TQ_EUNSUPPORTED, "level %d / bits %d: levels 1..10, bits 1..4", level, bits);
  return tq_polar_codebook_fp64(level, bits, centroids, thresholds);
}

tq_status tq_ctx_create_srht(const tq_spec *spec, const int8_t *rot_signs, const int8_t *qjl_signs,
                             int32_t device, tq_ctx **out) {
  g_err[0] = 0;
  if (!out) return tq_fail(TQ_EINVAL, "out is NULL");
  *out = nullptr;
  tq_status st = check_spec(spec);
  if (st != TQ_OK) return st;
  if (!qjl_signs) return tq_fail(TQ_EINVAL, "qjl_signs is NULL");
  const int d = spec->d, m = spec->qjl_m;
  if (m <= 0 || m > d)
    return tq_fail(TQ_EUNSUPPORTED, "structured QJL: qjl_m=%d must be in [32, d=%d]", m, d);
  for (int j = 0; j < d; ++j)
    if (qjl_signs[j] != 1 && qjl_signs[j] != -1)
      return tq_fail(TQ_EINVAL, "qjl_signs[%d] = %d: must be +1 or -1", j, (int)qjl_signs[j]);
  // S[i][j] = H[i][j] D2[j], H the unnormalised Sylvester Hadamard matrix: (-1)^popcount(i & j)
  float *S = new (std::nothrow) float[(size_t)m * d];
  if (!S) return tq_fail(TQ_ENOMEM, "host allocation failed");
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < d; ++j) S[(size_t)i * d + j] = (__builtin_popcount((unsigned)(i & j)) & 1) ? -qjl_signs[j] : qjl_signs[j];
  st = ctx_create(spec, rot_signs, S, qjl_signs, false, device, out);
  delete[] S;
  return st;
}

tq_status tq_ctx_destroy(tq_ctx *ctx) {
  if (!ctx) return TQ_OK;
  int cur = -1;
  cudaGetDevice(&cur);
  cudaSetDevice(ctx->device);
  cudaFree(ctx->dev_signs);
  cudaFree(ctx->dev_S);
  cudaFree(ctx->dev_St);
  cudaFree(ctx->dev_qjl_signs);
  cudaFree(ctx->dev_polar);
  if (cur >= 0) cudaSetDevice(cur);
  delete ctx;
  return TQ_OK;
}

tq_status tq_ctx_layout(const tq_ctx *ctx, int64_t *code_bytes, int64_t *sign_bytes) {
  g_err[0] = 0;
  tq_status st = check_ctx(ctx, "ctx");
  if (st != TQ_OK) return st;
  if (code_bytes) *code_bytes = ctx->code_bytes;
  if (sign_bytes) *sign_bytes = ctx->sign_bytes;
  return TQ_OK;
}

tq_status tq_encode_workspace_size(const tq_ctx *ctx, int64_t n, size_t *bytes) {
  g_err[0] = 0;
  tq_status st = check_ctx(ctx, "ctx");
  if (st != TQ_OK) return st;
  if (!bytes) return tq_fail(TQ_EINVAL, "bytes is NULL");
  if (n < 0) return tq_fail(TQ_EINVAL, "n < 0");
  const int64_t rows = n < kEncodeChunk ? n : kEncodeChunk;
  const bool fused = !ctx->k.polar && ((n <= kFusedEncodeMaxRows && ctx->spec.d >= 128) || ctx->k.srht);
  *bytes = (ctx->spec.qjl_m > 0 && !fused) ? (size_t)(rows * ctx->spec.d * 4) : 0;
  return TQ_OK;
}

tq_status tq_encode_kv(const tq_ctx *ctx, const void *x, tq_dtype dtype, int64_t n, int64_t ld,
                       const int64_t *slots, tq_packed out, void *ws, size_t ws_bytes,
                       void *stream) {
  g_err[0] = 0;
  tq_status st = check_ctx(ctx, "ctx");
  if (st != TQ_OK) return st;
  if (n < 0) return tq_fail(TQ_EINVAL, "n < 0");
  if (n == 0) return TQ_OK;
  if (!x) return tq_fail(TQ_EINVAL, "x is NULL");
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_EINVAL, "unknown dtype %d", (int)dtype);
  if (ld < ctx->spec.d) return tq_fail(TQ_EINVAL, "ld=%lld < d=%d", (long long)ld, ctx->spec.d);
  const int esz = dtype == TQ_F32 ? 4 : 2;
  if (!aligned16(x) || (ld * esz) % 16 != 0)
    return tq_fail(TQ_EINVAL, "x must be 16-byte aligned with a row stride that is a multiple of 16 bytes");
  if (slots && (reinterpret_cast<uintptr_t>(slots) & 7u))
    return tq_fail(TQ_EINVAL, "slots not 8-byte aligned");
  st = check_packed(ctx, out, slots ? 0 : n, "out", true);
  if (st != TQ_OK) return st;
  size_t need = 0;
  tq_encode_workspace_size(ctx, n, &need);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws)))
    return tq_fail(TQ_EINVAL, "workspace: %zu bytes (16-byte aligned) needed, %zu given", need, ws_bytes);
  DeviceScope dev_scope;
  st = dev_scope.enter(ctx->device);
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool qjl = ctx->spec.qjl_m > 0;
  if (ctx->k.polar) {
    // PolarQuant first stage; with a QJL stage the residual rows pass through the workspace
    for (int64_t r0 = 0; r0 < n; r0 += kEncodeChunk) {
      const int64_t rows = (n - r0) < kEncodeChunk ? (n - r0) : kEncodeChunk;
      const char *xr = static_cast<const char *>(x) + r0 * ld * esz;
      const int64_t *sl = slots ? slots + r0 : nullptr;
      tq_packed o = out;
      if (!slots) {
        o.codes = static_cast<char *>(out.codes) + r0 * ctx->code_bytes;
        o.norm = norm_at(ctx, out.norm, r0);
        if (qjl) {
          o.signs = static_cast<char *>(out.signs) + r0 * ctx->sign_bytes;
          o.rnorm = norm_at(ctx, out.rnorm, r0);
        }
        o.capacity = out.capacity - r0;
      }
      cudaError_t e = launch_encode_polar(ctx->k, xr, dtype, rows, ld, sl, o.capacity, static_cast<uint32_t *>(o.codes),
                                          o.norm, qjl ? o.rnorm : nullptr, qjl ? static_cast<float *>(ws) : nullptr, s);
      if (e == cudaSuccess && qjl)
        e = launch_project(ctx->k, PROJ_SIGNS, static_cast<const float *>(ws), rows, sl, o.capacity,
                           static_cast<uint32_t *>(o.signs), nullptr, s);
      if (e != cudaSuccess) return tq_cuda_check(e, "polar encode launch");
    }
    return TQ_OK;
  }
  if (n > kFusedEncodeMaxRows && encode_tpr_eligible(ctx->k, slots, dtype)) {
    // bulk rows at d = 128: one row per thread
    const int64_t nt = encode_tpr_rows(ctx->k, n);
    cudaError_t e = launch_encode_tpr(ctx->k, x, dtype, nt, ld, slots, out.capacity, static_cast<uint32_t *>(out.codes),
                                      out.norm, out.rnorm, static_cast<uint32_t *>(out.signs), s);
    if (e != cudaSuccess || nt == n) return tq_cuda_check(e, "encode launch");
    // the ragged tail of a token-block layout (rows nt.. go to slots nt..; nt is a whole block)
    e = launch_rotate(ctx->k, ROT_ENCODE, static_cast<const char *>(x) + nt * ld * esz, dtype, n - nt, ld, nullptr,
                      out.capacity - nt, static_cast<uint32_t *>(out.codes) + nt * (ctx->code_bytes / 4), norm_at(ctx, out.norm, nt),
                      nullptr, nullptr, s);
    return tq_cuda_check(e, "encode launch");
  }
  if (qjl && ctx->k.srht) {
    // structured QJL: the kernel transforms the residual itself (Walsh-Hadamard), any batch size
    cudaError_t e = launch_rotate(ctx->k, ROT_ENCODE, x, dtype, n, ld, slots, out.capacity,
                                  static_cast<uint32_t *>(out.codes), out.norm, out.rnorm, nullptr, s,
                                  static_cast<uint32_t *>(out.signs));
    return tq_cuda_check(e, "encode launch");
  }
  if (qjl && n <= kFusedEncodeMaxRows && ctx->spec.d >= 128) {
    // one launch: rotate, quantize, pack, project and pack the signs
    cudaError_t e = launch_rotate(ctx->k, ROT_ENCODE, x, dtype, n, ld, slots, out.capacity,
                                  static_cast<uint32_t *>(out.codes), out.norm, out.rnorm, nullptr, s,
                                  static_cast<uint32_t *>(out.signs));
    return tq_cuda_check(e, "fused encode launch");
  }
  for (int64_t r0 = 0; r0 < n; r0 += kEncodeChunk) {
    const int64_t rows = (n - r0) < kEncodeChunk ? (n - r0) : kEncodeChunk;
    const char *xr = static_cast<const char *>(x) + r0 * ld * esz;
    const int64_t *sl = slots ? slots + r0 : nullptr;
    // without a slot map, chunk rows land at slots r0 + i: shift the packed base pointers
    tq_packed o = out;
    if (!slots) {
      o.codes = static_cast<char *>(out.codes) + r0 * ctx->code_bytes;
      o.norm = norm_at(ctx, out.norm, r0);
      if (qjl) {
        o.signs = static_cast<char *>(out.signs) + r0 * ctx->sign_bytes;
        o.rnorm = norm_at(ctx, out.rnorm, r0);
      }
      o.capacity = out.capacity - r0;
    }
    cudaError_t e = launch_rotate(ctx->k, ROT_ENCODE, xr, dtype, rows, ld, sl, o.capacity,
                                  static_cast<uint32_t *>(o.codes), o.norm, qjl ? o.rnorm : nullptr,
                                  qjl ? static_cast<float *>(ws) : nullptr, s);
    if (e != cudaSuccess) return tq_cuda_check(e, "encode rotation launch");
    if (qjl) {
      e = launch_project(ctx->k, PROJ_SIGNS, static_cast<const float *>(ws), rows, sl, o.capacity,
                         static_cast<uint32_t *>(o.signs), nullptr, s);
      if (e != cudaSuccess) return tq_cuda_check(e, "QJL projection launch");
    }
  }
  return TQ_OK;
}

tq_status tq_scores_workspace_size(const tq_ctx *ctx, int32_t nq, size_t *bytes) {
  g_err[0] = 0;
  tq_status st = check_ctx(ctx, "ctx");
  if (st != TQ_OK) return st;
  if (!bytes) return tq_fail(TQ_EINVAL, "bytes is NULL");
  if (nq < 0) return tq_fail(TQ_EINVAL, "nq < 0");
  *bytes = query_prep_bytes(ctx, nq);
  return TQ_OK;
}

tq_status tq_scores(const tq_ctx *ctx, const void *q, tq_dtype dtype, int32_t nq, tq_packed keys,
                    int64_t n, float *out, void *ws, size_t ws_bytes, void *stream) {
  g_err[0] = 0;
  tq_status st = check_ctx(ctx, "ctx");
  if (st != TQ_OK) return st;
  if (nq < 0 || n < 0) return tq_fail(TQ_EINVAL, "nq < 0 or n < 0");
  if (nq == 0 || n == 0) return TQ_OK;
  if (!q || !out) return tq_fail(TQ_EINVAL, "q/out is NULL");
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_EINVAL, "unknown dtype %d", (int)dtype);
  if (!aligned16(q) || !aligned16(out)) return tq_fail(TQ_EINVAL, "q/out not 16-byte aligned");
  if (ctx->spec.layout != TQ_LAYOUT_ROWS) return tq_fail(TQ_EUNSUPPORTED, "tq_scores needs TQ_LAYOUT_ROWS");
  st = check_packed(ctx, keys, n, "keys", true);
  if (st != TQ_OK) return st;
  const size_t need = query_prep_bytes(ctx, nq);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return tq_fail(TQ_EINVAL, "workspace: %zu bytes (16-byte aligned) needed, %zu given", need, ws_bytes);
  DeviceScope dev_scope;
  st = dev_scope.enter(ctx->device);
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float *qr = static_cast<float *>(ws);
  float *p = reinterpret_cast<float *>(static_cast<char *>(ws) + tq_align_up((int64_t)nq * ctx->spec.d * 4, 256));
  st = prep_queries(ctx, q, dtype, nq, qr, p, s);
  if (st != TQ_OK) return st;
  if (ctx->k.polar) return tq_cuda_check(launch_scores_polar(ctx->k, qr, p, nq, keys, n, out, s), "scores launch");
  return tq_cuda_check(launch_scores(ctx->k, qr, p, nq, keys, n, out, s), "scores launch");
}

static tq_status check_attn(const tq_ctx *kctx, const tq_ctx *vctx, const tq_attn_desc *desc) {
  tq_status st = check_ctx(kctx, "kctx");
  if (st != TQ_OK) return st;
  st = check_ctx(vctx, "vctx");
  if (st != TQ_OK) return st;
  if (!desc) return tq_fail(TQ_EINVAL, "desc is NULL");
  if (kctx->spec.d != vctx->spec.d)
    return tq_fail(TQ_EUNSUPPORTED, "K and V contexts differ in d (%d vs %d)", kctx->spec.d, vctx->spec.d);
  if (vctx->spec.qjl_m != 0)
    return tq_fail(TQ_EUNSUPPORTED, "the V context must be MSE-only (qjl_m == 0)");
  if (kctx->spec.layout != TQ_LAYOUT_ROWS)
    return tq_fail(TQ_EUNSUPPORTED, "the K context must use TQ_LAYOUT_ROWS");
  if (vctx->spec.layout == TQ_LAYOUT_BLOCK16 && !desc->block_table && (desc->ctx_stride % 16) != 0)
    return tq_fail(TQ_EINVAL, "TQ_LAYOUT_BLOCK16 values need ctx_stride to be a multiple of 16");
  if (vctx->spec.layout == TQ_LAYOUT_BLOCK16 && desc->block_table && (desc->block_size % 16) != 0)
    return tq_fail(TQ_EINVAL, "TQ_LAYOUT_BLOCK16 values need block_size to be a multiple of 16");
  if (desc->batch < 0 || desc->n_q_heads <= 0 || desc->n_kv_heads <= 0)
    return tq_fail(TQ_EINVAL, "batch/n_q_heads/n_kv_heads");
  if (desc->n_q_heads % desc->n_kv_heads != 0)
    return tq_fail(TQ_EINVAL, "n_q_heads %% n_kv_heads != 0");
  const int g = desc->n_q_heads / desc->n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8)
    return tq_fail(TQ_EUNSUPPORTED, "group size %d: must be 1, 2, 4 or 8", g);
  if (desc->max_seq_len < 0) return tq_fail(TQ_EINVAL, "max_seq_len < 0");
  if (!desc->seq_lens && desc->batch > 0) return tq_fail(TQ_EINVAL, "seq_lens is NULL");
  if (desc->block_table) {
    if (desc->block_size <= 0 || desc->max_blocks <= 0)
      return tq_fail(TQ_EINVAL, "paged: block_size and max_blocks must be > 0");
    if ((int64_t)desc->max_blocks * desc->block_size < desc->max_seq_len)
      return tq_fail(TQ_EINVAL, "paged: max_blocks * block_size < max_seq_len");
  } else {
    if (desc->ctx_stride < desc->max_seq_len)
      return tq_fail(TQ_EINVAL, "contiguous: ctx_stride < max_seq_len");
  }
  st = check_packed(kctx, desc->k, 0, "desc->k", true);
  if (st != TQ_OK) return st;
  return check_packed(vctx, desc->v, 0, "desc->v", false);
}

tq_status tq_attend_workspace_size(const tq_ctx *kctx, const tq_ctx *vctx, const tq_attn_desc *desc,
                                   size_t *bytes) {
  g_err[0] = 0;
  tq_status st = check_attn(kctx, vctx, desc);
  if (st != TQ_OK) return st;
  if (!bytes) return tq_fail(TQ_EINVAL, "bytes is NULL");
  const AttnPlan plan = attn_plan(*desc, kctx->k, vctx->k);
  const int64_t nq = (int64_t)desc->batch * desc->n_q_heads;
  *bytes = query_prep_bytes(kctx, nq) + attn_partials_bytes(*desc, plan, kctx->spec.d);
  return TQ_OK;
}

tq_status tq_attend_decode(const tq_ctx *kctx, const tq_ctx *vctx, const tq_attn_desc *desc,
                           const void *q, tq_dtype dtype, float *out, void *ws, size_t ws_bytes,
                           void *stream) {
  g_err[0] = 0;
  tq_status st = check_attn(kctx, vctx, desc);
  if (st != TQ_OK) return st;
  if (desc->batch == 0) return TQ_OK;
  if (!q || !out) return tq_fail(TQ_EINVAL, "q/out is NULL");
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_EINVAL, "unknown dtype %d", (int)dtype);
  if (!aligned16(q) || !aligned16(out)) return tq_fail(TQ_EINVAL, "q/out not 16-byte aligned");
  size_t need = 0;
  tq_attend_workspace_size(kctx, vctx, desc, &need);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return tq_fail(TQ_EINVAL, "workspace: %zu bytes (16-byte aligned) needed, %zu given", need, ws_bytes);
  DeviceScope dev_scope;
  st = dev_scope.enter(kctx->device);
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nq = (int64_t)desc->batch * desc->n_q_heads;
  float *qr = static_cast<float *>(ws);
  float *p = reinterpret_cast<float *>(static_cast<char *>(ws) + tq_align_up(nq * kctx->spec.d * 4, 256));
  float *part = reinterpret_cast<float *>(static_cast<char *>(ws) + query_prep_bytes(kctx, nq));
  const AttnPlan plan = attn_plan(*desc, kctx->k, vctx->k);
  if (!plan.fast) {  // the tensor-core path rotates and projects the queries itself
    st = prep_queries(kctx, q, dtype, nq, qr, p, s);
    if (st != TQ_OK) return st;
  }
  return tq_cuda_check(launch_attend(kctx->k, vctx->k, *desc, plan, q, (int)dtype, qr, p, part, out, s),
                       "attention launch");
}

tq_status tq_decode_step_workspace_size(const tq_ctx *kctx, const tq_ctx *vctx, const tq_attn_desc *desc,
                                        int64_t n_new, size_t *bytes) {
  g_err[0] = 0;
  if (!bytes) return tq_fail(TQ_EINVAL, "bytes is NULL");
  if (n_new < 0 || n_new > kFusedEncodeMaxRows) return tq_fail(TQ_EINVAL, "n_new must be in [0, %lld]",
                                                               (long long)kFusedEncodeMaxRows);
  size_t att = 0, ek = 0, ev = 0;
  tq_status st = tq_attend_workspace_size(kctx, vctx, desc, &att);
  if (st != TQ_OK) return st;
  tq_encode_workspace_size(kctx, n_new, &ek);
  tq_encode_workspace_size(vctx, n_new, &ev);
  *bytes = att + (size_t)tq_align_up((int64_t)(ek > ev ? ek : ev), 256);
  return TQ_OK;
}

tq_status tq_decode_step(const tq_ctx *kctx, const tq_ctx *vctx, const tq_attn_desc *desc, const void *k_new,
                         const void *v_new, tq_dtype kv_dtype, int64_t n_new, const int64_t *new_slots,
                         const void *q, tq_dtype q_dtype, float *out, void *ws, size_t ws_bytes, void *stream) {
  g_err[0] = 0;
  size_t need = 0;
  tq_status st = tq_decode_step_workspace_size(kctx, vctx, desc, n_new, &need);
  if (st != TQ_OK) return st;
  if (desc->batch == 0) return TQ_OK;
  if (n_new > 0 && (!k_new || !v_new || !new_slots)) return tq_fail(TQ_EINVAL, "k_new/v_new/new_slots is NULL");
  if (!q || !out) return tq_fail(TQ_EINVAL, "q/out is NULL");
  if ((kv_dtype != TQ_F32 && kv_dtype != TQ_BF16) || (q_dtype != TQ_F32 && q_dtype != TQ_BF16))
    return tq_fail(TQ_EINVAL, "unknown dtype");
  if ((k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new)) || !aligned16(q) || !aligned16(out))
    return tq_fail(TQ_EINVAL, "k_new/v_new/q/out not 16-byte aligned");
  if (new_slots && (reinterpret_cast<uintptr_t>(new_slots) & 7u)) return tq_fail(TQ_EINVAL, "new_slots not 8-byte aligned");
  if (!ws || ws_bytes < need || !aligned16(ws))
    return tq_fail(TQ_EINVAL, "workspace: %zu bytes (16-byte aligned) needed, %zu given", need, ws_bytes);
  const AttnPlan plan = attn_plan(*desc, kctx->k, vctx->k);
  const int esz = kv_dtype == TQ_F32 ? 4 : 2;
  if (!plan.fast || (kctx->spec.d * esz) % 16 != 0) {
    // general path: the three calls in order; the encode workspace follows the attention's
    size_t att = 0;
    tq_attend_workspace_size(kctx, vctx, desc, &att);
    void *ews = static_cast<char *>(ws) + att;
    const size_t eb = ws_bytes - att;
    if (n_new > 0) {
      st = tq_encode_kv(kctx, k_new, kv_dtype, n_new, kctx->spec.d, new_slots, desc->k, ews, eb, stream);
      if (st != TQ_OK) return st;
      st = tq_encode_kv(vctx, v_new, kv_dtype, n_new, vctx->spec.d, new_slots, desc->v, ews, eb, stream);
      if (st != TQ_OK) return st;
    }
    return tq_attend_decode(kctx, vctx, desc, q, q_dtype, out, ws, att, stream);
  }
  DeviceScope dev_scope;
  st = dev_scope.enter(kctx->device);
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nq = (int64_t)desc->batch * desc->n_q_heads;
  float *part = reinterpret_cast<float *>(static_cast<char *>(ws) + query_prep_bytes(kctx, nq));
  void *extra = reinterpret_cast<char *>(part) +
                tq_align_up((int64_t)sizeof(float) * desc->batch * desc->n_q_heads * plan.splits * (kctx->spec.d + 4), 256);
  cudaError_t e = launch_decode_step_fast(kctx->k, vctx->k, *desc, plan, k_new, v_new, (int)kv_dtype, n_new, new_slots,
                                          q, (int)q_dtype, extra, part, plan.fused ? out : nullptr, s);
  if (e != cudaSuccess) return tq_cuda_check(e, "decode step launch");
  if (plan.fused) return TQ_OK;
  return tq_cuda_check(launch_attend_combine(vctx->k, *desc, plan, part, out, s), "combine launch");
}

tq_status tq_search_workspace_size(const tq_ctx *ctx, int32_t nq, int64_t n, int32_t k, size_t *bytes) {
  g_err[0] = 0;
  // the supported range of k is checked first (it does not depend on the context)
  if (k < 1) return tq_fail(TQ_EINVAL, "k=%d: must be >= 1", k);
  if (k > kSearchMaxK) return tq_fail(TQ_EUNSUPPORTED, "k=%d: at most %d", k, kSearchMaxK);
  tq_status st = check_ctx(ctx, "ctx");
  if (st != TQ_OK) return st;
  if (!bytes) return tq_fail(TQ_EINVAL, "bytes is NULL");
  if (nq < 0 || n < 0) return tq_fail(TQ_EINVAL, "nq/n");
  if (k > kSearchWarpMaxK) {  // the large-k scan only
    const int64_t cands = (int64_t)nq * search_bigk_shards(nq, n) * k;
    *bytes = query_prep_bytes(ctx, nq) + (size_t)tq_align_up(cands * 4, 256) + (size_t)tq_align_up(cands * 8, 256);
    return TQ_OK;
  }
  // room for either scan: the tensor-core one also needs 16-byte aligned norms, known only at the call
  const bool tc = search_tc_eligible(ctx->k, nq, k);
  const bool mma = search_mma_eligible(ctx->k) && nq <= kSearchMmaMaxQ;
  const int shards = std::max({search_plan(nq, n, k).shards, mma ? search_mma_shards(ctx->k, nq, n, k) : 1,
                               tc ? search_tc_shards(nq, n) : 1});
  const int64_t cands = (int64_t)nq * shards * k;
  *bytes = query_prep_bytes(ctx, nq) + (size_t)tq_align_up(cands * 4, 256) + (size_t)tq_align_up(cands * 8, 256) +
           std::max(mma ? search_mma_frag_bytes(ctx->k, nq) : 0, tc ? search_tc_ws_bytes(ctx->k, nq) : 0);
  return TQ_OK;
}

tq_status tq_search_topk(const tq_ctx *ctx, const void *q, tq_dtype dtype, int32_t nq, tq_packed db,
                         int64_t n, int32_t k, float *out_scores, int64_t *out_idx, void *ws,
                         size_t ws_bytes, void *stream) {
  g_err[0] = 0;
  if (k < 1) return tq_fail(TQ_EINVAL, "k=%d: must be >= 1", k);
  if (k > kSearchMaxK) return tq_fail(TQ_EUNSUPPORTED, "k=%d: at most %d", k, kSearchMaxK);
  tq_status st = check_ctx(ctx, "ctx");
  if (st != TQ_OK) return st;
  if (nq < 0 || n < 0) return tq_fail(TQ_EINVAL, "nq < 0 or n < 0");
  if (k > n) return tq_fail(TQ_EINVAL, "k=%d must be in [1, n=%lld]", k, (long long)n);
  if (nq == 0) return TQ_OK;
  if (!q || !out_scores || !out_idx) return tq_fail(TQ_EINVAL, "q/out is NULL");
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_EINVAL, "unknown dtype %d", (int)dtype);
  if (!aligned16(q) || !aligned16(out_scores) || !aligned16(out_idx))
    return tq_fail(TQ_EINVAL, "q/out not 16-byte aligned");
  if (ctx->spec.layout != TQ_LAYOUT_ROWS) return tq_fail(TQ_EUNSUPPORTED, "tq_search_topk needs TQ_LAYOUT_ROWS");
  st = check_packed(ctx, db, n, "db", true);
  if (st != TQ_OK) return st;
  size_t need = 0;
  tq_search_workspace_size(ctx, nq, n, k, &need);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return tq_fail(TQ_EINVAL, "workspace: %zu bytes (16-byte aligned) needed, %zu given", need, ws_bytes);
  DeviceScope dev_scope;
  st = dev_scope.enter(ctx->device);
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k > kSearchWarpMaxK) {
    // large k: CUDA-core scan with shared-memory top-k buffers, then their merge
    const int shards = search_bigk_shards(nq, n);
    const int64_t cands = (int64_t)nq * shards * k;
    char *w = static_cast<char *>(ws);
    float *qr = reinterpret_cast<float *>(w);
    float *p = reinterpret_cast<float *>(w + tq_align_up((int64_t)nq * ctx->spec.d * 4, 256));
    w += query_prep_bytes(ctx, nq);
    float *cs = reinterpret_cast<float *>(w);
    int64_t *ci = reinterpret_cast<int64_t *>(w + tq_align_up(cands * 4, 256));
    st = prep_queries(ctx, q, dtype, nq, qr, p, s);
    if (st != TQ_OK) return st;
    return tq_cuda_check(launch_search_bigk(ctx->k, shards, qr, p, nq, db, n, k, cs, ci, out_scores, out_idx, s),
                         "search launch");
  }
  // scan: tcgen05 (many queries), else the bit-plane mma.sync scan, else CUDA cores
  const bool tc = search_tc_eligible(ctx->k, nq, k);
  const bool mma = !tc && search_mma_eligible(ctx->k) && nq <= kSearchMmaMaxQ && aligned16(db.norm) &&
                   aligned16(db.rnorm) && !ctx->k.norm16;  // that scan copies fp32 norms in bulk
  const SearchPlan plan = search_plan(nq, n, k);
  const int shards = tc ? search_tc_shards(nq, n) : mma ? search_mma_shards(ctx->k, nq, n, k) : plan.shards;
  const int64_t cands = (int64_t)nq * shards * k;
  char *w = static_cast<char *>(ws);
  float *qr = reinterpret_cast<float *>(w);
  float *p = reinterpret_cast<float *>(w + tq_align_up((int64_t)nq * ctx->spec.d * 4, 256));
  w += query_prep_bytes(ctx, nq);
  float *cs = reinterpret_cast<float *>(w);
  int64_t *ci = reinterpret_cast<int64_t *>(w + tq_align_up(cands * 4, 256));
  void *fragws = w + tq_align_up(cands * 4, 256) + tq_align_up(cands * 8, 256);
  st = prep_queries(ctx, q, dtype, nq, qr, p, s);
  if (st != TQ_OK) return st;
  if (tc || mma) {
    // tensor-core scan (bit-plane MMAs), then the same merge of the shards' candidates
    cudaError_t e = tc ? launch_search_tc(ctx->k, shards, qr, p, nq, db, n, k, fragws, cs, ci, s)
                       : launch_search_mma(ctx->k, shards, qr, p, nq, db, n, k, fragws, cs, ci, s);
    if (e == cudaSuccess) e = launch_search_merge(nq, shards, k, cs, ci, out_scores, out_idx, s);
    return tq_cuda_check(e, "search launch");
  }
  return tq_cuda_check(launch_search(ctx->k, plan, qr, p, nq, db, n, k, cs, ci, out_scores, out_idx, s),
                       "search launch");
}

}  // extern "C"
