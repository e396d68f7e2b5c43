// profiler.cu -- optional per-kernel timing with CUDA events (host code).
// When a plan's profiling is on, every launch is bracketed by two events
// recorded on the launch's own stream; deltakv_profile_collect sums them.
#include <cstdio>
#include <cstring>
#include <vector>

#include "internal.h"

namespace dkv {

struct Profiler {
  struct Rec { int kid; cudaEvent_t a, b; };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
  ~Profiler() {
    for (auto& r : recs) { cudaEventDestroy(r.a); cudaEventDestroy(r.b); }
    for (auto e : pool) cudaEventDestroy(e);
  }
};

const char* kernel_name(int id) {
  static const char* names[KID_COUNT] = {
      "refpack", "candidates_simt", "candidates_tc", "encode_simt", "encode_tc", "reconstruct",
      "decode_ref", "decode_prep", "decode_stream_simt", "decode_stream_tc", "decode_combine", "decode_final",
      "append_refs", "append_rows", "sparse_attend", "sparse_merge", "sparse_select"};
  return (id >= 0 && id < KID_COUNT) ? names[id] : "?";
}

ProfScope::ProfScope(const Plan& p, cudaStream_t s, int k) : prof(p.prof), st(s), kid(k), slot(-1) {
  if (!prof) return;
  cudaEvent_t a = prof->get(), b = prof->get();
  if (!a || !b) { prof = nullptr; return; }
  cudaEventRecord(a, st);
  prof->recs.push_back({kid, a, b});
  slot = (int)prof->recs.size() - 1;
}

ProfScope::~ProfScope() {
  if (prof && slot >= 0) cudaEventRecord(prof->recs[slot].b, st);
}

Profiler* profiler_create() { return new Profiler(); }
void profiler_destroy(Profiler* p) { delete p; }

int profiler_collect(Profiler* p, deltakv_kernel_time* out, int n_max) {
  double ms[KID_COUNT] = {0};
  int cnt[KID_COUNT] = {0};
  bool fail = false;
  for (auto& r : p->recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      fail = true;
    ms[r.kid] += t;
    cnt[r.kid] += 1;
    p->pool.push_back(r.a);
    p->pool.push_back(r.b);
  }
  p->recs.clear();
  if (fail) return -1;
  int n = 0;
  for (int k = 0; k < KID_COUNT && n < n_max; ++k) {
    if (!cnt[k]) continue;
    std::memset(out[n].name, 0, sizeof(out[n].name));
    std::strncpy(out[n].name, kernel_name(k), sizeof(out[n].name) - 1);
    out[n].launches = cnt[k];
    out[n].total_ms = ms[k];
    ++n;
  }
  return n;
}

}  // namespace dkv
