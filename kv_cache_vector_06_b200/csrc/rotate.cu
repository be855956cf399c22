// Encode stage 1 and query rotation: one warp (or a group of lanes for d < 128) per vector.
//
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
#include "rotate_device.cuh"

namespace {

template <int D>
__global__ void __launch_bounds__(kRotThreads)
rotate_kernel(TqConsts c, int mode, const void *__restrict__ x, int dtype, int64_t n, int64_t ld,
              const int64_t *__restrict__ slots, int64_t capacity, uint32_t *__restrict__ codes,
              void *__restrict__ norm, void *__restrict__ rnorm, float *__restrict__ resid,
              uint32_t *__restrict__ fsigns) {
  extern __shared__ __align__(16) float sS[];
  rotate_rows<D>(c, mode, x, dtype, n, ld, slots, capacity, codes, norm, rnorm, resid, fsigns,
                 (int64_t)blockIdx.x, sS);
}

template <int D>
cudaError_t launch_rotate_d(const TqConsts &c, RotateMode mode, const void *x, tq_dtype dtype,
                            int64_t n, int64_t ld, const int64_t *slots, int64_t capacity,
                            uint32_t *codes, void *norm, void *rnorm, float *resid,
                            uint32_t *fsigns, cudaStream_t st) {
  constexpr int VPB = (kRotThreads / 32) * RotLayout<D>::VPW;  // vectors per block
  const int64_t blocks = (n + VPB - 1) / VPB;
  const int kind = mode == ROT_ENCODE ? TQK_ROTATE_ENCODE : TQK_ROTATE_QUERY;
  const size_t smem = (D == 128 && fsigns != nullptr && c.m == 128 && !c.srht) ? sizeof(float) * 128 * 132 : 0;
  if (smem) {
    cudaError_t e0 = tq_smem_limit(reinterpret_cast<const void *>(rotate_kernel<D>), (int)smem);
    if (e0 != cudaSuccess) return e0;
  }
  tq_prof_begin(kind, st);
  rotate_kernel<D><<<(unsigned)blocks, kRotThreads, smem, st>>>(c, (int)mode, x, (int)dtype, n, ld, slots,
                                                                capacity, codes, norm, rnorm, resid, fsigns);
  tq_prof_end(kind, st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rotate(const TqConsts &c, RotateMode mode, const void *x, tq_dtype dtype,
                          int64_t n, int64_t ld, const int64_t *slots, int64_t capacity,
                          uint32_t *codes, void *norm, void *rnorm, float *resid,
                          cudaStream_t st, uint32_t *fsigns) {
  if (n <= 0) return cudaSuccess;
  switch (c.d) {
#define TQ_ROT_CASE(DD) \
  case DD: return launch_rotate_d<DD>(c, mode, x, dtype, n, ld, slots, capacity, codes, norm, rnorm, resid, fsigns, st);
    TQ_ROT_CASE(8) TQ_ROT_CASE(16) TQ_ROT_CASE(32) TQ_ROT_CASE(64)
    TQ_ROT_CASE(128) TQ_ROT_CASE(256) TQ_ROT_CASE(512) TQ_ROT_CASE(1024)
#undef TQ_ROT_CASE
    default: return cudaErrorInvalidValue;
  }
}

// The device flags of this translation unit's kernels (see tq_device_status).
TQ_DEVICE_FLAGS_ACCESSOR(rotate_device_flags)
