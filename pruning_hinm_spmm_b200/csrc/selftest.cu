// Diagnostic: exercises the bounded-wait path every pipelined kernel of the library relies
// on.  Thread 0 waits on an mbarrier that nothing arrives at; after the limit it records
// HINM_ERR_DEVICE_TIMEOUT and raises the CTA's abort flag, which releases a second thread
// waiting on another barrier (as the other roles of a pipelined kernel are released).
// Nothing faults, traps or hangs: the kernel returns after about `limit_ns`.
#include <cuda_runtime.h>

#include "hinm_internal.h"
#include "ptx.cuh"

namespace hinm {

__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns, int* status) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&bars[0]), 1);
    ptx::mbar_init(ptx::smem_u32(&bars[1]), 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_wait_for(ptx::smem_u32(&bars[0]), 0, status, abort, limit_ns);  // times out
  } else if (threadIdx.x == 32) {
    // released by the abort flag; its own limit is twice as long, so a missing abort
    // would show as a second (distinguishable) late return, never as a hang
    ptx::mbar_wait_for(ptx::smem_u32(&bars[1]), 0, status, abort, 2 * limit_ns);
  }
  __syncthreads();
}

cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, int* status,
                                         cudaStream_t s) {
  wait_timeout_selftest_kernel<<<1, 64, 0, s>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace hinm
