// Launch accounting: a process-wide count of the library's kernel launches and, when
// enabled, CUDA events recorded around each launch on its stream (per-kernel device time).
#include <atomic>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "gdn.h"
#include "gdn_launch.h"

namespace gdn {
namespace {
struct Rec {
  const char* name;
  cudaEvent_t a, b;
};
std::mutex g_mu;
std::vector<Rec> g_recs;
std::atomic<int> g_on{0};
std::atomic<long long> g_launches{0};
}  // namespace

ProfScope::ProfScope(const char* name, cudaStream_t s) : name_(name), s_(s) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (g_on.load(std::memory_order_relaxed)) {
    cudaEventCreate(&a_);
    cudaEventCreate(&b_);
    cudaEventRecord(a_, s_);
    active_ = true;
  }
}

ProfScope::~ProfScope() {
  if (!active_) return;
  cudaEventRecord(b_, s_);
  std::lock_guard<std::mutex> g(g_mu);
  g_recs.push_back({name_, a_, b_});
}

}  // namespace gdn

using namespace gdn;

extern "C" {

int64_t gdn_launch_count(void) { return g_launches.load(); }

int gdn_profile(int enable) {
  g_on.store(enable ? 1 : 0);
  return GDN_OK;
}

int64_t gdn_profile_read(char* buf, size_t cap) {
  std::vector<Rec> recs;
  {
    std::lock_guard<std::mutex> g(g_mu);
    recs.swap(g_recs);
  }
  std::map<std::string, std::pair<long long, double>> agg;
  int rc = GDN_OK;
  for (auto& r : recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      rc = GDN_ERR_CUDA;
    auto& e = agg[r.name];
    e.first += 1;
    e.second += ms;
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  std::string s = "{";
  bool first = true;
  for (auto& kv : agg) {
    char tmp[256];
    snprintf(tmp, sizeof tmp, "%s\"%s\": [%lld, %.6f]", first ? "" : ", ", kv.first.c_str(),
             kv.second.first, kv.second.second);
    s += tmp;
    first = false;
  }
  s += "}";
  if (rc != GDN_OK) return -rc;
  if (buf && cap > 0) {
    const size_t n = s.size() < cap - 1 ? s.size() : cap - 1;
    memcpy(buf, s.data(), n);
    buf[n] = 0;
  }
  return (int64_t)s.size();
}

}  // extern "C"
