// Failure-detection self-test: proves on the device that a barrier wait which
// can never complete ends by itself, records SINKATTN_ERR_TIMEOUT and lets the
// kernel return (no trap, no hang), using the same bounded wait as the
// attention kernels.
#include "internal.h"

namespace sk {
namespace {

__global__ void wait_selftest_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival that never comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, &abort_flag, status);
}

}  // namespace

int launch_wait_selftest(int* status, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace sk
