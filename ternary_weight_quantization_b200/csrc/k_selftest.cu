// Self-test of the bounded device waits every pipeline kernel uses: one warp
// waits on an mbarrier that nothing ever arrives on. The wait gives up after
// its time bound, records the timeout in the device error word and returns,
// so the host can read the failure and keep using the context.
#include <cuda_runtime.h>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

__global__ void selftest_wait_kernel(int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, &abort_flag, err);  // no arrival ever comes
}

}  // namespace

cudaError_t launch_selftest_timeout(int* err, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

}  // namespace bl
