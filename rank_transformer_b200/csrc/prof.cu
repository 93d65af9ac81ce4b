// Optional per-launch profiler: CUDA events around eager launches, summed
// per operation name.  Graph replays are not instrumented.
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"

namespace fsvd {

namespace {

struct Pending {
  std::string name;
  double bytes, flops;
  cudaEvent_t start, stop;
};
struct Stat {
  long long count = 0;
  double ms = 0.0, bytes = 0.0, flops = 0.0;
};

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;
std::map<std::string, Stat> g_stats;
cudaEvent_t g_open = nullptr;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

void resolve_locked() {
  for (auto& p : g_pending) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p.start, p.stop) == cudaSuccess) {
      Stat& s = g_stats[p.name];
      s.count += 1;
      s.ms += ms;
      s.bytes += p.bytes;
      s.flops += p.flops;
    }
    g_pool.push_back(p.start);
    g_pool.push_back(p.stop);
  }
  g_pending.clear();
}

}  // namespace

bool prof_active(cudaStream_t s) {
  if (!g_on.load(std::memory_order_relaxed)) return false;
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &st) != cudaSuccess) return false;
  return st == cudaStreamCaptureStatusNone;
}

void prof_begin(cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_open = take_event();
  cudaEventRecord(g_open, s);
}

void prof_end(const LaunchTag& tag, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_mu);
  cudaEvent_t stop = take_event();
  cudaEventRecord(stop, s);
  g_pending.push_back(Pending{tag.name, tag.bytes, tag.flops, g_open, stop});
  g_open = nullptr;
  if (g_pending.size() > 4096) {  // bound the number of live events
    cudaEventSynchronize(stop);
    resolve_locked();
  }
}

}  // namespace fsvd

extern "C" {

int flashsvd_profile_enable(int on) {
  fsvd::g_on.store(on != 0);
  return FLASHSVD_OK;
}

int flashsvd_profile_report(char* buf, int buflen, int reset) {
  using namespace fsvd;
  std::lock_guard<std::mutex> lock(g_mu);
  FSVD_CUDA(cudaDeviceSynchronize());
  resolve_locked();
  std::string out;
  char line[256];
  for (auto& kv : g_stats) {
    snprintf(line, sizeof(line), "%s %lld %.6f %.6e %.6e\n", kv.first.c_str(), kv.second.count,
             kv.second.ms, kv.second.bytes, kv.second.flops);
    out += line;
  }
  if (reset) g_stats.clear();
  if (!buf || buflen <= 0) return (int)out.size() + 1;
  snprintf(buf, (size_t)buflen, "%s", out.c_str());
  return FLASHSVD_OK;
}

}  // extern "C"
