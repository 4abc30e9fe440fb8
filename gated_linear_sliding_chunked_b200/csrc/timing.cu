// Opt-in per-launch timing: when enabled on a host thread, every kernel the
// library launches from that thread is bracketed by a pair of CUDA events
// recorded on the launch's own stream.  Benchmarks read the elapsed times
// back with lz_timing_read.  Off by default; costs nothing when off.
#include <cstring>
#include <string>
#include <vector>

#include "../../include/lizard.h"
#include "kernels.h"

namespace lz {
namespace {

struct Rec {
  const char* name;
  cudaEvent_t a, b;
};

thread_local bool g_on = false;
thread_local std::string g_only;  // empty: every launch; else only launches of this name
thread_local std::vector<Rec> g_recs;
thread_local std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

ScopedTiming::ScopedTiming(const char* name, cudaStream_t s)
    : s_(s), on_(g_on && (g_only.empty() || g_only == name)) {
  if (!on_) return;
  name_ = name;
  a_ = take_event();
  b_ = take_event();
  if (!a_ || !b_) {
    on_ = false;
    return;
  }
  cudaEventRecord(a_, s_);
}

ScopedTiming::~ScopedTiming() {
  if (!on_) return;
  cudaEventRecord(b_, s_);
  g_recs.push_back(Rec{name_, a_, b_});
}

}  // namespace lz

extern "C" {

int lz_timing_enable(int on) {
  lz::g_on = on != 0;
  return 0;
}

int lz_timing_only(const char* name) {
  lz::g_only = name ? name : "";
  return 0;
}

int lz_timing_read(char* names, size_t name_stride, float* ms, int max_records) {
  int n = 0;
  for (auto& r : lz::g_recs) {
    if (n < max_records) {
      float t = -1.f;
      if (cudaEventSynchronize(r.b) == cudaSuccess) cudaEventElapsedTime(&t, r.a, r.b);
      if (ms) ms[n] = t;
      if (names && name_stride > 0) {
        std::strncpy(names + (size_t)n * name_stride, r.name, name_stride - 1);
        names[(size_t)n * name_stride + name_stride - 1] = '\0';
      }
    } else {
      cudaEventSynchronize(r.b);
    }
    lz::g_pool.push_back(r.a);
    lz::g_pool.push_back(r.b);
    ++n;
  }
  lz::g_recs.clear();
  return n;
}

}  // extern "C"
