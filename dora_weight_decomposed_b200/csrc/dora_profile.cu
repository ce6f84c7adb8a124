// Kernel-level timing inside the library. When started, every kernel the
// library launches is bracketed by a pair of CUDA events recorded on the
// launch stream, and launched without programmatic dependent launch (so that
// it cannot start under its predecessor's events); during stream capture the events become event-record nodes of
// the graph, so each replay of the graph re-times the same kernels. Reading
// waits for the events and reports each launch's duration. Meant for
// benchmarks on one host thread; off by default and free when off.
#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "dora_internal.h"

namespace dora {

namespace {

struct Rec {
  const char* name;
  cudaEvent_t start;
  cudaEvent_t stop;
};

struct Profiler {
  std::mutex mu;
  bool on = false;
  int capacity = 0;
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;  // 2 * capacity events
};

Profiler& prof() {
  static Profiler p;
  return p;
}

cudaError_t record(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  if (cs == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  return cudaEventRecord(ev, st);
}

}  // namespace

bool profiling_on() {
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  return p.on;
}

ProfRange::ProfRange(const char* name, cudaStream_t st) : st_(st), idx_(-1) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  if (!p.on || (int)p.recs.size() >= p.capacity) return;
  const int i = (int)p.recs.size();
  Rec r{name, p.pool[2 * i], p.pool[2 * i + 1]};
  if (record(r.start, st) != cudaSuccess) return;
  p.recs.push_back(r);
  idx_ = i;
}

ProfRange::~ProfRange() {
  if (idx_ < 0) return;
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  record(p.recs[idx_].stop, st_);
}

}  // namespace dora

using namespace dora;

extern "C" {

dora_status_t dora_profile_start(int capacity) {
  if (capacity <= 0 || capacity > (1 << 20)) {
    set_error("capacity out of range");
    return DORA_EINVAL;
  }
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  for (cudaEvent_t e : p.pool) cudaEventDestroy(e);
  p.pool.clear();
  p.recs.clear();
  p.pool.resize(2 * (size_t)capacity, nullptr);
  for (auto& e : p.pool) {
    cudaError_t err = cudaEventCreate(&e);
    if (err != cudaSuccess) {
      p.on = false;
      return cuda_status(err, "dora_profile_start");
    }
  }
  p.capacity = capacity;
  p.on = true;
  return DORA_OK;
}

dora_status_t dora_profile_stop(void) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  p.on = false;
  return DORA_OK;
}

int dora_profile_count(void) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  return (int)p.recs.size();
}

dora_status_t dora_profile_read(dora_profile_record_t* out, int capacity, int* n_out) {
  if (!out || !n_out || capacity < 0) {
    set_error("dora_profile_read: bad arguments");
    return DORA_EINVAL;
  }
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  const int n = std::min<int>(capacity, (int)p.recs.size());
  for (int i = 0; i < n; ++i) {
    cudaError_t e = cudaEventSynchronize(p.recs[i].stop);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p.recs[i].start, p.recs[i].stop);
    if (e != cudaSuccess) return cuda_status(e, "dora_profile_read");
    out[i].name = p.recs[i].name;
    out[i].ms = ms;
  }
  *n_out = n;
  return DORA_OK;
}

}  // extern "C"
