// Self-test of the device error path: one thread waits, with an iteration
// limit, on a shared-memory mbarrier that nothing arrives at. The wait gives
// up, ORs kDevErrWaitTimeout into the device error word and the kernel returns
// normally, the way every kernel of the library ends a wait that cannot
// complete (no trap, no fault, the context stays usable).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "vq_device.cuh"

namespace vq {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t max_iters) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) (void)mbar_wait_bounded(&bar, 0, max_iters);
}

}  // namespace

inline cudaError_t launch_wait_timeout(uint32_t max_iters, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(max_iters);
  return cudaGetLastError();
}

}  // namespace vq
