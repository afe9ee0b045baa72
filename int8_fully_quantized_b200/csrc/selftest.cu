// Self-test of the device-side failure path: every wait of the library's kernels is bounded (ptx.cuh,
// mbar_wait) and reports through the status word that jf_device_status reads. This kernel waits on an
// mbarrier that nothing ever arrives on, with a short limit, so that the path can be exercised on a
// GPU without any fault: the wait gives up, raises the timeout bit and the kernel returns.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace jf {

__global__ void __launch_bounds__(32) wait_selftest_kernel(unsigned int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0u;
    fence_mbar_init();
  }
  __syncwarp();
  // phase 0 of a fresh barrier never completes: nothing arrives on it
  if (threadIdx.x == 0) mbar_wait(&bar, 0u, &abort_flag, status, limit_ns);
}

cudaError_t launch_wait_selftest(unsigned int* status, unsigned long long limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace jf
