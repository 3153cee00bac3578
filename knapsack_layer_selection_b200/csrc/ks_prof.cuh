// Launch accounting of the library: how many kernels of each kind were enqueued,
// their algorithmic FLOPs and bytes, and (when timing is on) their device time
// measured with CUDA events recorded on the launching stream.
#pragma once

#include "ks_common.cuh"

namespace ks {

enum KernelKind {
  KK_RMSNORM = 0,
  KK_GEMM_Q,
  KK_GEMM_O,
  KK_GEMM_GATEUP,
  KK_GEMM_DOWN,
  KK_ROPE,
  KK_SWIGLU,
  KK_ATTN,
  KK_SELECT,
  KK_RECONSTRUCT,
  KK_TPT,
  KK_BROADCAST,
  KK_ROPE_TABLE,
  KK_DEDUP,
  KK_GATHER,
  KK_DEDUP_VERIFY,
  KK_GEMM_KV,
  KK_COUNT
};

const char* kernel_kind_name(int k);

// Brackets the launches of one kernel kind.  Counts them always; records a
// pair of events around them when timing is enabled.
class ProfScope {
 public:
  ProfScope(int kind, cudaStream_t st, double flops, double bytes, int n_launches = 1);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  int kind_;
  cudaStream_t st_;
  int slot_;
};

}  // namespace ks
