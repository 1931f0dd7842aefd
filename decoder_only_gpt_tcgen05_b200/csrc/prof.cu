// Launch counter and optional per-launch CUDA-event timing (see Prof in host.cuh).
#include <mutex>
#include <vector>

#include "gpt_ops.h"
#include "host.cuh"

namespace gptk {

namespace {
struct Rec {
  int kind;
  double flops, bytes;
  cudaEvent_t a, b;
};
std::mutex g_mu;
bool g_on = false;
unsigned long long g_launches = 0;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t get_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

Prof::Prof(int kind, double flops, double bytes, cudaStream_t st) : idx_(-1), st_(st) {
  std::lock_guard<std::mutex> lk(g_mu);
  ++g_launches;
  if (!g_on) return;
  Rec r{kind, flops, bytes, get_event(), get_event()};
  cudaEventRecord(r.a, st);
  g_recs.push_back(r);
  idx_ = static_cast<int>(g_recs.size()) - 1;
}

Prof::~Prof() {
  if (idx_ < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (idx_ < static_cast<int>(g_recs.size())) cudaEventRecord(g_recs[idx_].b, st_);
}

}  // namespace gptk

using namespace gptk;

extern "C" {

GPT_API unsigned long long gpt_launch_count(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_launches;
}

GPT_API int gpt_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (Rec& r : g_recs) {
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  g_on = true;
  return 0;
}

GPT_API int gpt_profile_stop(int max_kinds, double* ms, long long* count, double* flops, double* bytes) {
  set_error(ST_OK, "");
  std::lock_guard<std::mutex> lk(g_mu);
  g_on = false;
  for (int k = 0; k < max_kinds; ++k) {
    if (ms) ms[k] = 0;
    if (count) count[k] = 0;
    if (flops) flops[k] = 0;
    if (bytes) bytes[k] = 0;
  }
  for (Rec& r : g_recs) {
    GPTK_CUDA(cudaEventSynchronize(r.b));
    float t = 0.f;
    GPTK_CUDA(cudaEventElapsedTime(&t, r.a, r.b));
    if (r.kind < max_kinds) {
      if (ms) ms[r.kind] += t;
      if (count) count[r.kind] += 1;
      if (flops) flops[r.kind] += r.flops;
      if (bytes) bytes[r.kind] += r.bytes;
    }
  }
  return PK_COUNT;
}

}  // extern "C"
