// Per-kernel event timing registry (see profile.cuh).
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/moe.h"
#include "profile.cuh"

namespace moe {
namespace {

struct Pending {
  std::string name;
  cudaEvent_t a, b;
};

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_free;
struct Agg {
  long launches = 0;
  double ms = 0.0;
};
std::map<std::string, Agg> g_agg;

cudaEvent_t grab() {
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

}  // namespace

bool profile_on() { return g_on.load(std::memory_order_relaxed); }

int profile_begin(const char* name, cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_mu);
  Pending p{name, grab(), grab()};
  cudaEventRecord(p.a, st);
  g_pending.push_back(p);
  return (int)g_pending.size() - 1;
}

void profile_end(int token, cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (token >= 0 && token < (int)g_pending.size()) cudaEventRecord(g_pending[token].b, st);
}

}  // namespace moe

extern "C" {

moe_status moe_profile_enable(int on) {
  moe::g_on.store(on != 0);
  return MOE_OK;
}

moe_status moe_profile_collect(moe_profile_entry* out, int32_t cap, int32_t* n_out) {
  if (!n_out || cap < 0 || (cap > 0 && !out)) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(moe::g_mu);
  for (auto& p : moe::g_pending) {
    if (cudaEventSynchronize(p.b) != cudaSuccess) return MOE_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess) return MOE_ERR_CUDA;
    auto& a = moe::g_agg[p.name];
    a.launches += 1;
    a.ms += ms;
    moe::g_free.push_back(p.a);
    moe::g_free.push_back(p.b);
  }
  moe::g_pending.clear();
  int n = 0;
  for (auto& kv : moe::g_agg) {
    if (n < cap) {
      std::memset(&out[n], 0, sizeof(moe_profile_entry));
      std::strncpy(out[n].name, kv.first.c_str(), sizeof(out[n].name) - 1);
      out[n].launches = kv.second.launches;
      out[n].total_ms = kv.second.ms;
    }
    ++n;
  }
  *n_out = n;
  moe::g_agg.clear();
  return MOE_OK;
}

}  // extern "C"
