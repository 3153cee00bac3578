// Diagnostics of the device-side failure handling: one mbarrier wait that
// nothing completes, bounded by the same routine every tensor-core kernel uses.
#include "ks_sm100.cuh"

namespace ks {
namespace {

__global__ void wait_probe_kernel(int32_t* status, unsigned long long* waited_ns,
                                  unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(sm100::smem_u32(&bar), 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_ns();
    // nothing arrives on `bar`, so phase 0 never completes
    const bool ok = sm100::mbar_wait(sm100::smem_u32(&bar), 0, &abort_flag, status, limit_ns);
    if (waited_ns) *waited_ns = global_ns() - t0;
    if (ok) raise_status(status, KS_ERR_INTERNAL);
  }
}

}  // namespace
}  // namespace ks

using namespace ks;

extern "C" KS_API ks_status ks_check_bounded_wait(uint32_t limit_us, int32_t* status,
                                                  uint64_t* waited_ns, ks_stream_t stream) {
  if (!status) return fail(KS_ERR_INVALID_ARG, "check_bounded_wait: status is NULL");
  if (limit_us < 1 || limit_us > 2000000)
    return fail(KS_ERR_INVALID_ARG, "check_bounded_wait: limit must be 1 us .. 2 s");
  wait_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(
      status, (unsigned long long*)waited_ns, (unsigned long long)limit_us * 1000ull);
  KS_LAUNCH_CHECK();
  return KS_OK;
}
