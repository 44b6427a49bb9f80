// Self test of the bounded device wait: one thread waits on an mbarrier that
// nothing ever arrives on, gives up after `wait_ns`, records the timeout in the
// status word and returns.  It exercises the same mbar_wait used by the tensor
// core kernels, without faulting, trapping or hanging the device.
#include "common.cuh"
#include "kernels.h"

namespace dn {
namespace {

__global__ void wait_selftest_kernel(unsigned int* status, unsigned long long wait_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtl w{&abort_flag, status, wait_ns};
    (void)mbar_wait(smem_u32(&bar), 0, w);  // phase 0 never completes
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned int* status, long long wait_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, (unsigned long long)wait_ns);
  return cudaGetLastError();
}

}  // namespace dn
