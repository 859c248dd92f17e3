// Self-test of the bounded pipeline wait: one thread waits, through the same
// mbar_wait every pipeline uses, on an mbarrier that nothing ever completes.
// The wait gives up at its limit (about two seconds), records
// MISA_DEVERR_TIMEOUT in the error word and the kernel returns, so the
// context stays usable.  Nothing faults, traps or hangs.
#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

__global__ void wait_timeout_selftest_kernel(uint32_t* err, uint32_t* result) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) *result = mbar_wait(&bar, 0, err) ? 1u : 0u;  // phase 0 never completes
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(uint32_t* err, uint32_t* result, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err, result);
  return cudaGetLastError();
}

}  // namespace misa
