// Per-launch kernel timing: event pairs around chosen kernels, with the
// launch's algorithmic work (include/gq.h, "Per-launch kernel timing").
#include <mutex>
#include <vector>

#include "gq_internal.h"

namespace gq {

std::atomic<uint32_t> g_timer_mask{0};

namespace {

struct Record {
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  int kind = -1;
  double work = 0.0;
};

std::mutex g_mu;
std::vector<Record> g_recs;
size_t g_used = 0;
int g_dev = -1;
bool g_active = false;

cudaError_t record(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) == cudaSuccess && cap == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  return cudaEventRecord(e, st);
}

}  // namespace

int timer_begin_slow(gq_kernel k, cudaStream_t st) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!(g_timer_mask.load() & (1u << k)) || g_used >= g_recs.size()) return -1;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != g_dev) return -1;
  Record &r = g_recs[g_used];
  if (record(r.e0, st) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  r.kind = k;
  return static_cast<int>(g_used++);
}

void timer_end_slow(int slot, cudaStream_t st, double work) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (slot < 0 || static_cast<size_t>(slot) >= g_recs.size()) return;
  Record &r = g_recs[slot];
  if (record(r.e1, st) != cudaSuccess) {
    cudaGetLastError();
    r.kind = -1;
    return;
  }
  r.work = work;
}

}  // namespace gq

using namespace gq;

extern "C" gq_status gq_kernel_timer_start(uint32_t mask, int32_t capacity) {
  clear_error();
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_active) return fail(GQ_ERR_ARG, "a kernel timer session is already active");
  if (capacity <= 0) return fail(GQ_ERR_ARG, "capacity must be positive");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return check_launch("cudaGetDevice");
  g_recs.assign(static_cast<size_t>(capacity), Record{});
  for (Record &r : g_recs) {
    if (cudaEventCreate(&r.e0) != cudaSuccess || cudaEventCreate(&r.e1) != cudaSuccess) {
      const gq_status s = check_launch("cudaEventCreate");
      for (Record &q : g_recs) {
        if (q.e0) cudaEventDestroy(q.e0);
        if (q.e1) cudaEventDestroy(q.e1);
      }
      g_recs.clear();
      return s;
    }
  }
  g_used = 0;
  g_dev = dev;
  g_active = true;
  g_timer_mask.store(mask & ((1u << GQ_KERNEL_COUNT) - 1));
  return GQ_OK;
}

extern "C" gq_status gq_kernel_timer_stop(void) {
  g_timer_mask.store(0);
  return GQ_OK;
}

extern "C" int32_t gq_kernel_timer_read(int32_t *kind, float *ms, double *work, int32_t max) {
  clear_error();
  std::lock_guard<std::mutex> lock(g_mu);
  const int32_t n = static_cast<int32_t>(g_used);
  for (int32_t i = 0; i < n && i < max; ++i) {
    const Record &r = g_recs[i];
    float t = 0.0f;
    if (r.kind >= 0 && cudaEventElapsedTime(&t, r.e0, r.e1) != cudaSuccess) {
      check_launch("cudaEventElapsedTime");
      return -1;
    }
    if (kind) kind[i] = r.kind;
    if (ms) ms[i] = t;
    if (work) work[i] = r.work;
  }
  return n;
}

extern "C" gq_status gq_kernel_timer_release(void) {
  g_timer_mask.store(0);
  std::lock_guard<std::mutex> lock(g_mu);
  for (Record &r : g_recs) {
    if (r.e0) cudaEventDestroy(r.e0);
    if (r.e1) cudaEventDestroy(r.e1);
  }
  g_recs.clear();
  g_used = 0;
  g_active = false;
  return GQ_OK;
}
