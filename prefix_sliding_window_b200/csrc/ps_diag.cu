// Diagnostic kernel for the bounded waits every kernel of the library uses (ps_device.cuh,
// mbar_wait): a wait on a shared-memory barrier phase that nothing completes gives up after
// the wait limit, flags PS_DEV_TIMEOUT and lets the kernel return.
#include <cuda_runtime.h>

#include "ps_device.cuh"

namespace ps {
namespace {

// One expected arrival, none made: the barrier's first phase never completes.
__global__ void wait_timeout_kernel(int32_t* __restrict__ status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, status);
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout(int32_t* status, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace ps
