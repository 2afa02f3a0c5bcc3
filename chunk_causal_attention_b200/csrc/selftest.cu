// Diagnostic entry point: checks that a device-side wait of this library ends
// and reports instead of hanging.  One thread waits, with the same bounded
// mbarrier wait the attention kernel uses, on a barrier phase that nothing
// completes (or, as a positive control, that the thread completes itself first).
#include "common.cuh"
#include "sm100.cuh"

namespace cca {

__global__ void selftest_bounded_wait_kernel(int32_t *status, long long budget, int arrive_first) {
  using namespace sm100;
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (arrive_first) mbar_arrive(&bar);
    const bool ok = mbar_wait(&bar, 0, &abort_flag, budget);
    *status = ok ? CCA_DEV_OK : CCA_DEV_TIMEOUT;
  }
}

}  // namespace cca

using namespace cca;

extern "C" cca_status cca_selftest_bounded_wait(int32_t *dev_status, int64_t budget_cycles, int32_t arrive_first,
                                                cca_stream_t stream) {
  if (!dev_status || (reinterpret_cast<uintptr_t>(dev_status) & 3))
    return fail(CCA_ERR_INVALID_ARG, "cca_selftest_bounded_wait: dev_status must be a 4-byte aligned device pointer");
  if (budget_cycles < 1 || budget_cycles > 4000000000LL)
    return fail(CCA_ERR_INVALID_ARG, "cca_selftest_bounded_wait: budget must be in [1, 4e9] cycles");
  selftest_bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(dev_status, budget_cycles,
                                                                                    arrive_first);
  return launched("selftest_bounded_wait_kernel");
}
