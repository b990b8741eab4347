// rvq_api.cu -- status strings, the launch counter, the distance-GEMM profiling hooks and the
// host-side fault injection switch.
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "rvq.h"
#include "rvq_host.h"

namespace rvq {

static std::atomic<int64_t> g_launches{0};

void note_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int device_sm_count(int *sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RVQ_ERR_CUDA;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return RVQ_ERR_CUDA;
  return RVQ_OK;
}

int injected_fault(const char *entry) {
  static const std::vector<std::pair<std::string, int>> faults = [] {
    std::vector<std::pair<std::string, int>> v;
    const char *e = getenv("RVQ_FAULT");
    std::string spec = e ? e : "";
    size_t pos = 0;
    while (pos < spec.size()) {
      size_t end = spec.find(',', pos);
      if (end == std::string::npos) end = spec.size();
      const std::string item = spec.substr(pos, end - pos);
      const size_t colon = item.rfind(':');
      if (colon != std::string::npos) {
        const int code = atoi(item.c_str() + colon + 1);
        if (code < 0 && code >= RVQ_ERR_TIMEOUT) v.emplace_back(item.substr(0, colon), code);
      }
      pos = end + 1;
    }
    return v;
  }();
  for (const auto &f : faults)
    if (f.first == entry) return f.second;
  return 0;
}

namespace {
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;  // even = start, odd = end
  std::vector<int> levels;        // RVQ levels covered by each bracketed launch
  size_t used = 0;                // events handed out since enable
};
Profiler &prof() {
  static Profiler p;
  return p;
}
cudaEvent_t take_event() {
  Profiler &p = prof();
  if (p.used == p.pool.size()) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    p.pool.push_back(e);
  }
  return p.pool[p.used++];
}
}  // namespace

bool profiling_enabled() { return prof().on; }

void profile_begin(cudaStream_t s) {
  Profiler &p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.on) return;
  if (p.used % 2 != 0) return;  // unmatched begin; keep pairs aligned
  cudaEvent_t e = take_event();
  if (e) cudaEventRecord(e, s);
}

void profile_end(cudaStream_t s, int levels) {
  Profiler &p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.on) return;
  if (p.used % 2 != 1) return;
  cudaEvent_t e = take_event();
  if (e) {
    cudaEventRecord(e, s);
    p.levels.resize(p.used / 2);
    p.levels.back() = levels;
  }
}

}  // namespace rvq

extern "C" {

const char *rvq_status_str(int status) {
  switch (status) {
    case RVQ_OK: return "RVQ_OK";
    case RVQ_ERR_ARG: return "RVQ_ERR_ARG: invalid argument";
    case RVQ_ERR_UNSUPPORTED: return "RVQ_ERR_UNSUPPORTED: shape outside the supported range";
    case RVQ_ERR_WORKSPACE: return "RVQ_ERR_WORKSPACE: workspace missing or too small";
    case RVQ_ERR_CUDA: return "RVQ_ERR_CUDA: a CUDA call failed";
    case RVQ_ERR_ID_RANGE: return "RVQ_ERR_ID_RANGE: id outside [0, K)";
    case RVQ_ERR_TIMEOUT: return "RVQ_ERR_TIMEOUT: an encode pipeline wait timed out";
    default: return "unknown rvq status";
  }
}

int64_t rvq_launch_count(void) { return rvq::g_launches.load(std::memory_order_relaxed); }

int rvq_profile_enable(int enable) {
  rvq::Profiler &p = rvq::prof();
  std::lock_guard<std::mutex> g(p.mu);
  p.on = enable != 0;
  p.used = 0;
  p.levels.clear();
  return RVQ_OK;
}

int rvq_profile_read(int64_t *gemm_launches, double *gemm_ms) {
  if (!gemm_launches || !gemm_ms) return RVQ_ERR_ARG;
  rvq::Profiler &p = rvq::prof();
  std::lock_guard<std::mutex> g(p.mu);
  double total = 0.0;
  int64_t n = 0;
  for (size_t i = 0; i + 1 < p.used; i += 2) {
    if (cudaEventSynchronize(p.pool[i + 1]) != cudaSuccess) return RVQ_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p.pool[i], p.pool[i + 1]) != cudaSuccess) return RVQ_ERR_CUDA;
    total += ms;
    n += i / 2 < p.levels.size() ? p.levels[i / 2] : 1;
  }
  *gemm_launches = n;
  *gemm_ms = total;
  return RVQ_OK;
}

}  // extern "C"
