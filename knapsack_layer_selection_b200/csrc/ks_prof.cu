// Launch accounting (see ks_prof.cuh) and its C ABI: ks_profile_start/stop.
#include <string.h>

#include <mutex>
#include <vector>

#include "ks_prof.cuh"

namespace ks {

namespace {

struct Pending {
  int kind;
  cudaEvent_t a, b;
};

struct Profiler {
  std::mutex mu;
  bool timing = false;
  long long launches[KK_COUNT] = {};
  double flops[KK_COUNT] = {};
  double bytes[KK_COUNT] = {};
  double ms[KK_COUNT] = {};
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> pool;

  cudaEvent_t get_event() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};

Profiler& prof() {
  static Profiler p;
  return p;
}

}  // namespace

const char* kernel_kind_name(int k) {
  static const char* names[KK_COUNT] = {"rmsnorm", "gemm_q_rope", "gemm_o_residual",
                                        "gemm_gateup_swiglu", "gemm_down_residual", "rope",
                                        "swiglu", "attention", "select_bp", "reconstruct",
                                        "tpt_argmax", "init_states", "rope_table", "dedup",
                                        "gather", "dedup_verify", "gemm_kv_window"};
  return (k >= 0 && k < KK_COUNT) ? names[k] : "?";
}

ProfScope::ProfScope(int kind, cudaStream_t st, double flops, double bytes, int n_launches)
    : kind_(kind), st_(st), slot_(-1) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  p.launches[kind] += n_launches;
  p.flops[kind] += flops;
  p.bytes[kind] += bytes;
  if (!p.timing) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return;
  Pending pe{kind, p.get_event(), p.get_event()};
  if (!pe.a || !pe.b) return;
  if (cudaEventRecord(pe.a, st) != cudaSuccess) return;
  p.pending.push_back(pe);
  slot_ = (int)p.pending.size() - 1;
}

ProfScope::~ProfScope() {
  if (slot_ < 0) return;
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (slot_ < (int)p.pending.size()) cudaEventRecord(p.pending[slot_].b, st_);
}

}  // namespace ks

using namespace ks;

extern "C" {

KS_API ks_status ks_profile_start(int32_t timing) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  for (auto& pe : p.pending) {
    cudaEventSynchronize(pe.b);
    p.pool.push_back(pe.a);
    p.pool.push_back(pe.b);
  }
  p.pending.clear();
  memset(p.launches, 0, sizeof(p.launches));
  memset(p.flops, 0, sizeof(p.flops));
  memset(p.bytes, 0, sizeof(p.bytes));
  memset(p.ms, 0, sizeof(p.ms));
  p.timing = timing != 0;
  return KS_OK;
}

KS_API ks_status ks_profile_stop(ks_kernel_stat* stats, int32_t capacity, int32_t* n_kinds) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  for (auto& pe : p.pending) {
    if (cudaEventSynchronize(pe.b) != cudaSuccess) return fail(KS_ERR_CUDA, "profile: event sync");
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, pe.a, pe.b) == cudaSuccess) p.ms[pe.kind] += ms;
    p.pool.push_back(pe.a);
    p.pool.push_back(pe.b);
  }
  p.pending.clear();
  p.timing = false;
  int n = 0;
  for (int k = 0; k < KK_COUNT; ++k) {
    if (p.launches[k] == 0) continue;
    if (stats && n < capacity) {
      ks_kernel_stat& s = stats[n];
      memset(&s, 0, sizeof(s));
      strncpy(s.name, kernel_kind_name(k), sizeof(s.name) - 1);
      s.launches = p.launches[k];
      s.total_ms = p.ms[k];
      s.flops = p.flops[k];
      s.bytes = p.bytes[k];
    }
    ++n;
  }
  if (n_kinds) *n_kinds = n;
  return KS_OK;
}

}  // extern "C"
