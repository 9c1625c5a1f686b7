// Per-kernel-family timing with CUDA events (enabled on request; off by default).
#include "stats.h"

#include <mutex>
#include <vector>

namespace jolt {

namespace {
struct Pending {
  int fam;
  cudaEvent_t e0, e1;
  double flops, bytes, issued;
};
struct Acc {
  uint64_t launches = 0;
  double ms = 0, flops = 0, bytes = 0, issued = 0;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;
Acc g_acc[JOLT_K_COUNT];

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
}  // namespace

bool stats_on() {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_on;
}

StatScope::StatScope(int family, cudaStream_t st, double flops, double bytes, double issued)
    : fam_(family), st_(st), flops_(flops), bytes_(bytes), issued_(issued < 0.0 ? flops : issued) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on || family < 0) return;  // family < 0: not recorded (the caller's own scope covers it)
  e0_ = take_event();
  e1_ = take_event();
  if (e0_) cudaEventRecord(e0_, st_);
}

StatScope::~StatScope() {
  if (!e0_ || !e1_) return;
  cudaEventRecord(e1_, st_);
  std::lock_guard<std::mutex> lk(g_mu);
  g_pending.push_back(Pending{fam_, e0_, e1_, flops_, bytes_, issued_});
}

}  // namespace jolt

using namespace jolt;

extern "C" void jolt_stats_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_on = on != 0;
}

extern "C" jolt_status jolt_stats_read(jolt_kernel_stat* out, int32_t reset) {
  if (!out) return JOLT_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  for (const Pending& p : g_pending) {
    if (cudaEventSynchronize(p.e1) != cudaSuccess) return JOLT_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p.e0, p.e1) != cudaSuccess) return JOLT_ERR_CUDA;
    Acc& a = g_acc[p.fam];
    a.launches += 1;
    a.ms += ms;
    a.flops += p.flops;
    a.bytes += p.bytes;
    a.issued += p.issued;
    g_pool.push_back(p.e0);
    g_pool.push_back(p.e1);
  }
  g_pending.clear();
  for (int f = 0; f < JOLT_K_COUNT; ++f) {
    out[f].kernel = f;
    out[f].launches = g_acc[f].launches;
    out[f].ms = g_acc[f].ms;
    out[f].flops = g_acc[f].flops;
    out[f].bytes = g_acc[f].bytes;
    out[f].flops_issued = g_acc[f].issued;
    if (reset) g_acc[f] = Acc{};
  }
  return JOLT_OK;
}
