// Tensor-core GEMM (placeholder until the tcgen05 kernel lands): the bf16 path
// runs on the CUDA-core kernels.
#include "ks_tc.cuh"

namespace ks {

bool use_tensor_cores(const ks_model_desc* m) {
  (void)m;
  return false;
}

ks_status tc_gemm(const void*, const void*, const void*, void*, const float*, int, int, int, int,
                  const float2*, int, int, cudaStream_t) {
  return fail(KS_ERR_UNSUPPORTED, "tensor-core GEMM not built");
}

}  // namespace ks
