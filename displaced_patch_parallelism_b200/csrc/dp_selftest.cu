// dp_selftest.cu -- a kernel whose bounded wait nothing ever ends, so that the
// timeout path of the library's waits can be exercised without faulting or
// hanging the GPU.
//
// Every pipeline wait of the library's kernels is mbar_wait_limit (on an
// mbarrier in shared memory) or flag_wait_change (on a flag in global
// memory), each bounded by a wall-clock limit.  This kernel runs exactly those
// helpers on a barrier no thread arrives at, or on a flag no thread writes,
// with a caller-chosen limit: the wait runs out, records DP_ERR_TIMEOUT in the
// status word and the kernel returns normally.  No TMA copy or MMA is in
// flight, so nothing outlives the kernel.
#include "dp_common.cuh"
#include "dp_internal.h"

namespace dp {

// Never written: a flag wait on it can only end by its limit.
__device__ unsigned g_selftest_flag = 0u;

__global__ void selftest_wait_kernel(int kind, unsigned long long limit_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival completes a phase; none comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (kind == DP_SELFTEST_WAIT_MBARRIER)
      mbar_wait_limit(&bar, 0u, &abort_flag, status, limit_ns);
    else
      flag_wait_change(&g_selftest_flag, 0u, status, limit_ns);
  }
  __syncthreads();
}

}  // namespace dp

extern "C" {

int dp_selftest_bounded_wait(int kind, unsigned limit_us, void* stream) {
  if (kind != DP_SELFTEST_WAIT_MBARRIER && kind != DP_SELFTEST_WAIT_FLAG)
    return dp::set_error(DP_ERR_INVALID_ARG, "selftest: unknown wait kind %d", kind);
  if (limit_us < 1 || limit_us > 1000000u)
    return dp::set_error(DP_ERR_INVALID_ARG, "selftest: limit %u us outside [1, 1000000]", limit_us);
  int* status = dp::device_status_ptr();
  if (!status) return dp::set_error(DP_ERR_CUDA, "selftest: status word address unavailable");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  dp::selftest_wait_kernel<<<1, 32, 0, st>>>(kind, 1000ull * limit_us, status);
  return dp::cuda_check(cudaGetLastError(), "selftest launch");
}

}  // extern "C"
