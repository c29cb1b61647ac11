// Per-kernel timing for profiling runs (pisa_timing_start / pisa_timing_stop
// in include/pisa.h). While timing is on, each TimedLaunch records one CUDA
// event before its kernel and one after it, on the launching stream; stop
// waits for the events and sums the elapsed times per kernel name. The events
// are created on the device current at launch time and destroyed by stop.
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace pisa {
namespace {

struct Record {
  const char* name;
  cudaEvent_t start;
  cudaEvent_t stop;
  bool ok;
};

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<Record> g_records;

void release_all() {
  for (Record& r : g_records) {
    if (r.start) cudaEventDestroy(r.start);
    if (r.stop) cudaEventDestroy(r.stop);
  }
  g_records.clear();
}

}  // namespace

TimedLaunch::TimedLaunch(const char* name, cudaStream_t st) : slot_(-1), st_(st) {
  if (!g_on.load(std::memory_order_acquire)) return;
  Record r{name, nullptr, nullptr, false};
  if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) {
    if (r.start) cudaEventDestroy(r.start);
    if (r.stop) cudaEventDestroy(r.stop);
    return;
  }
  if (cudaEventRecord(r.start, st) != cudaSuccess) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
    return;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  slot_ = static_cast<int>(g_records.size());
  g_records.push_back(r);
}

TimedLaunch::~TimedLaunch() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lock(g_mu);
  if (slot_ < static_cast<int>(g_records.size())) {
    Record& r = g_records[slot_];
    r.ok = cudaEventRecord(r.stop, st_) == cudaSuccess;
  }
}

}  // namespace pisa

extern "C" pisa_status pisa_timing_start(void) {
  std::lock_guard<std::mutex> lock(pisa::g_mu);
  pisa::release_all();
  pisa::g_on.store(true, std::memory_order_release);
  return PISA_OK;
}

extern "C" int pisa_timing_stop(int max_kernels, const char** names, double* total_ms, int* launches) {
  using namespace pisa;
  g_on.store(false, std::memory_order_release);
  std::lock_guard<std::mutex> lock(g_mu);
  std::vector<const char*> nm;
  std::vector<double> ms;
  std::vector<int> cnt;
  int status = 0;
  for (Record& r : g_records) {
    float t = 0.f;
    if (!r.ok || cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) {
      status = -1;
      continue;
    }
    size_t i = 0;
    while (i < nm.size() && std::strcmp(nm[i], r.name) != 0) ++i;
    if (i == nm.size()) {
      nm.push_back(r.name);
      ms.push_back(0.0);
      cnt.push_back(0);
    }
    ms[i] += t;
    cnt[i] += 1;
  }
  release_all();
  if (status != 0) return -1;
  for (size_t i = 0; i < nm.size() && static_cast<int>(i) < max_kernels; ++i) {
    if (names) names[i] = nm[i];
    if (total_ms) total_ms[i] = ms[i];
    if (launches) launches[i] = cnt[i];
  }
  return static_cast<int>(nm.size());
}
