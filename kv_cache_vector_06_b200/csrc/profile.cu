// Optional per-kernel instrumentation: CUDA events recorded on the launching stream around each
// kernel, summed per kernel kind on request.  Off by default; not for use under stream capture.
#include <cstring>
#include <mutex>
#include <vector>

#include <map>
#include <utility>

#include "tq_internal.h"

namespace {

const char *kNames[TQK_COUNT] = {"rotate_encode", "qjl_project", "rotate_query", "query_project", "scores",
                                 "attend_split", "attend_combine", "search_scan", "search_merge",
                                 "attend_frag", "decode_prep", "encode_rows", "encode_qjl_tc"};

struct Pending {
  int kind;
  cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_free;
int64_t g_launches[TQK_COUNT];
double g_ms[TQK_COUNT];
thread_local cudaEvent_t t_open[TQK_COUNT];

cudaEvent_t take_event() {
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

void drain_locked() {
  for (const Pending &p : g_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
      g_ms[p.kind] += ms;
      g_launches[p.kind] += 1;
    }
    g_free.push_back(p.a);
    g_free.push_back(p.b);
  }
  g_pending.clear();
}

}  // namespace

bool tq_prof_on() {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_on;
}

void tq_prof_begin(int kind, cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on) return;
  cudaEvent_t e = take_event();
  if (e && cudaEventRecord(e, st) == cudaSuccess) {
    t_open[kind] = e;
  } else {
    if (e) g_free.push_back(e);
    t_open[kind] = nullptr;
  }
}

void tq_prof_end(int kind, cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on || !t_open[kind]) return;
  cudaEvent_t e = take_event();
  if (e && cudaEventRecord(e, st) == cudaSuccess) {
    g_pending.push_back({kind, t_open[kind], e});
  } else {
    g_free.push_back(t_open[kind]);
    if (e) g_free.push_back(e);
  }
  t_open[kind] = nullptr;
}

cudaError_t tq_smem_limit(const void *func, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, int> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  int &have = done[std::make_pair(func, dev)];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

extern "C" {

tq_status tq_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_on = on != 0;
  return TQ_OK;
}

tq_status tq_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  drain_locked();
  for (int i = 0; i < TQK_COUNT; ++i) {
    g_launches[i] = 0;
    g_ms[i] = 0.0;
  }
  return TQ_OK;
}

tq_status tq_profile_read(int32_t index, char *name, int32_t name_len, int64_t *launches, double *total_ms) {
  if (index < 0 || index >= TQK_COUNT) return tq_fail(TQ_EINVAL, "profile index %d out of range", index);
  std::lock_guard<std::mutex> lk(g_mu);
  drain_locked();
  if (name && name_len > 0) {
    std::strncpy(name, kNames[index], (size_t)name_len - 1);
    name[name_len - 1] = 0;
  }
  if (launches) *launches = g_launches[index];
  if (total_ms) *total_ms = g_ms[index];
  return TQ_OK;
}

}  // extern "C"
