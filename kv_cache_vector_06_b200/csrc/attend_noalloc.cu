// tq_attend_decode_noalloc: decode attention for callers that must not allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run attention: an inference engine
// that hands all device memory to its own pool at start-up and does not let extensions allocate,
// or a latency-critical decode loop where an allocator call may synchronize the device.  For
// them this entry point takes no workspace argument.  Its scratch space is one fixed array of
// device memory defined below; every GPU that loads the library holds that array until the
// process exits.
//
// Contract (also stated in include/tq.h):
//   - The first call on a device looks up the array's device address with cudaGetSymbolAddress
//     (with that device current) and caches it; make that first call before any stream capture.
//   - Requests whose workspace (tq_attend_workspace_size) exceeds TQ_NOALLOC_SCRATCH_BYTES are
//     rejected with TQ_EINVAL before anything is launched.
//   - Every call on a device shares the same array and leaves its contents behind.  Nothing in it
//     needs to start at zero: each call writes every scratch element it reads.  Calls whose work
//     overlaps on the GPU (different streams, or different host threads) race on the array; the
//     caller must order them (same stream, or events).
//   - No cudaMalloc, cudaFree or other allocating routine is called.
#include <mutex>

#include "tq_internal.h"

// Scratch for the allocation-free entry point (device memory, file scope).  In host code this
// name is only a stand-in for the symbol: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char tq_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on `device` (which must be current), looked up once.
tq_status scratch_address(int device, void **out) {
  if (device < 0 || device >= kMaxDevices)
    return tq_fail(TQ_EUNSUPPORTED, "device %d: the allocation-free entry point supports devices 0..%d",
                   device, kMaxDevices - 1);
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[device]) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, tq_noalloc_scratch);
    if (e != cudaSuccess) return tq_cuda_check(e, "cudaGetSymbolAddress(tq_noalloc_scratch)");
    g_scratch_addr[device] = p;
  }
  *out = g_scratch_addr[device];
  return TQ_OK;
}
}  // namespace

extern "C" tq_status tq_attend_decode_noalloc(const tq_ctx *kctx, const tq_ctx *vctx,
                                              const tq_attn_desc *desc, const void *q, tq_dtype dtype,
                                              float *out, void *stream) {
  size_t need = 0;
  tq_status st = tq_attend_workspace_size(kctx, vctx, desc, &need);
  if (st != TQ_OK) return st;
  if (need > (size_t)TQ_NOALLOC_SCRATCH_BYTES)
    return tq_fail(TQ_EINVAL,
                   "tq_attend_decode_noalloc: this request needs %zu bytes of scratch, more than the "
                   "%zu-byte static array; call tq_attend_decode with a workspace instead",
                   need, (size_t)TQ_NOALLOC_SCRATCH_BYTES);
  DeviceScope dev_scope;  // the caller's current device is restored on return
  st = dev_scope.enter(kctx->device);
  if (st != TQ_OK) return st;
  void *ws = nullptr;
  st = scratch_address(kctx->device, &ws);
  if (st != TQ_OK) return st;
  return tq_attend_decode(kctx, vctx, desc, q, dtype, out, ws, (size_t)TQ_NOALLOC_SCRATCH_BYTES, stream);
}
