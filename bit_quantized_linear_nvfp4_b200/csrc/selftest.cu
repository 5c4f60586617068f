// Self-test of the device-side failure path: every wait inside the library's
// kernels is bounded, and a wait that gives up sets the device error word that
// nvfp4_check reports, after which the kernel returns and the context stays
// usable.  wait_selftest_kernel runs that path on purpose: one thread waits,
// through the same bounded wait the GEMM kernels use, on an mbarrier that no
// thread ever arrives on, so the wait ends by its time limit.
#include <cstdint>

#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {

__global__ void wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
    // phase 0 of a fresh barrier never completes: nothing arrives
    mbar_wait_bounded(&bar, 0, nullptr, limit_ns);
  }
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns);
  return cudaGetLastError();
}

}  // namespace nvfp4
