// Internal helpers shared by the KnapSpec CUDA sources (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <initializer_list>
#include <string>

#include "../../include/knapspec.h"

namespace ks {

// ---------------------------------------------------------------- host errors
void set_error(const std::string& msg);
ks_status fail(ks_status s, const std::string& msg);

#define KS_CUDA_TRY(expr)                                                         \
  do {                                                                            \
    cudaError_t _e = (expr);                                                      \
    if (_e != cudaSuccess)                                                        \
      return ::ks::fail(KS_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(_e)); \
  } while (0)

#define KS_TRY(expr)                 \
  do {                               \
    ks_status _s = (expr);           \
    if (_s != KS_OK) return _s;      \
  } while (0)

#define KS_LAUNCH_CHECK() KS_CUDA_TRY(cudaGetLastError())

inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// Caller pointers that kernels move 16 bytes at a time (vector loads and
// stores, TMA) must be 16-byte aligned; checked at the C ABI before any launch
// so a misaligned view is an error code, not a misaligned access.  NULL passes.
inline ks_status check_aligned16(std::initializer_list<const void*> ptrs, const char* call) {
  for (const void* p : ptrs)
    if (p && (reinterpret_cast<uintptr_t>(p) & 15))
      return fail(KS_ERR_INVALID_ARG, std::string(call) + ": device pointers must be 16-byte aligned");
  return KS_OK;
}

// Runs `set` (a function-attribute setup returning ks_status) once per device
// for the call site owning `done`: function attributes are per device.  Two
// threads may both run it the first time, which is harmless.
template <typename F>
ks_status once_per_device(std::atomic<unsigned long long>& done, F&& set) {
  int dev = 0;
  KS_CUDA_TRY(cudaGetDevice(&dev));
  const unsigned long long bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load() & bit)) return KS_OK;
  KS_TRY(set());
  if (bit) done.fetch_or(bit);
  return KS_OK;
}

// ---------------------------------------------------------------- element types
template <typename T> struct Elem;
template <> struct Elem<float> {
  __device__ __forceinline__ static float to_f(float x) { return x; }
  __device__ __forceinline__ static float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  __device__ __forceinline__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Device status word: the first error code written wins.
__device__ __forceinline__ void raise_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// Nanosecond clock shared by all SMs; used to bound every spin-wait.
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// A bounded wait gives up after this long (legitimate waits last microseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

}  // namespace ks
