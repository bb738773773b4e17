// Optional per-kernel CUDA-event timing (benchmark instrumentation).
#include <cuda_runtime.h>
#include <string.h>

#include <map>
#include <string>
#include <vector>

#include "../../include/muse.h"
#include "kernels.h"

namespace muse {
namespace {

struct Rec {
  const char* name;
  cudaEvent_t a, b;
};

bool g_on = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e;
  cudaEventCreate(&e);
  return e;
}

}  // namespace

ProfScope::ProfScope(cudaStream_t s, const char* name) : st(s), slot(-1) {
  if (!g_on) return;
  Rec r{name, take_event(), take_event()};
  cudaEventRecord(r.a, st);
  g_recs.push_back(r);
  slot = (int)g_recs.size() - 1;
}

ProfScope::~ProfScope() {
  if (slot >= 0) cudaEventRecord(g_recs[slot].b, st);
}

}  // namespace muse

extern "C" {

void muse_profile_enable(int on) { muse::g_on = on != 0; }

int muse_profile_read(char* names, int name_stride, int* launches, double* ms, int cap) {
  using namespace muse;
  std::map<std::string, std::pair<int, double>> acc;
  std::vector<std::string> order;
  for (auto& r : g_recs) {
    cudaEventSynchronize(r.b);
    float t = 0.f;
    cudaEventElapsedTime(&t, r.a, r.b);
    auto it = acc.find(r.name);
    if (it == acc.end()) {
      order.push_back(r.name);
      acc[r.name] = {1, (double)t};
    } else {
      it->second.first += 1;
      it->second.second += t;
    }
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  int n = 0;
  for (auto& name : order) {
    if (n < cap) {
      if (names && name_stride > 0) {
        strncpy(names + (size_t)n * name_stride, name.c_str(), name_stride - 1);
        names[(size_t)n * name_stride + name_stride - 1] = 0;
      }
      if (launches) launches[n] = acc[name].first;
      if (ms) ms[n] = acc[name].second;
    }
    ++n;
  }
  return n;
}

}  // extern "C"
