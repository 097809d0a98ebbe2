// Self-test of the bounded waits: one CTA waits on an mbarrier that nothing
// arrives on, through the same bounded wait every kernel of the library
// uses, with a caller-given short limit.  The wait gives up, raises
// BASISKV_DEV_TIMEOUT in the device status word and the kernel returns, so
// a caller can check that a wait that cannot complete ends the kernel with
// a readable status and leaves the context usable.
#include <cuda_runtime.h>

#include "../../include/basiskv.h"
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {
namespace {

constexpr unsigned long long kMaxSelftestLimitNs = 1000000000ull;  // 1 s

__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns, unsigned int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Phase 0 completes only after one arrival, and no thread arrives.
  if (threadIdx.x == 0) mbar_wait(&bar, 0, status, limit_ns);
  __syncthreads();
}

}  // namespace
}  // namespace basiskv

extern "C" int basiskv_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  using namespace basiskv;
  if (limit_ns == 0 || limit_ns > kMaxSelftestLimitNs) return BASISKV_ERR_INVALID_ARG;
  unsigned int* status = device_status_ptr();
  if (!status) return BASISKV_ERR_CUDA;
  const cudaError_t e = launch_k(bounded_wait_selftest_kernel, dim3(1), dim3(32), 0,
                                 static_cast<cudaStream_t>(stream), false,
                                 (unsigned long long)limit_ns, status);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? BASISKV_OK
                                                               : BASISKV_ERR_LAUNCH_FAILED;
}
