// Diagnostics of the bounded waits every kernel of this library uses.
#include "internal.h"
#include "ptx.cuh"

namespace calibatt {
namespace {

using namespace ptx;

// One warp waits, through the kernels' bounded Waiter, on an mbarrier that
// nothing arrives on: after timeout_ns it records "timed out at wait point
// 15" in the status word and returns.  Exercises the failure path of every
// wait without a fault or a hang.
__global__ void bounded_wait_kernel(int32_t* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar_mem;
  __shared__ int abort_flag;
  const uint32_t bar = smem_addr(&bar_mem);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  const Waiter W{&abort_flag, status, timeout_ns};
  W.wait(bar, 0, 15);
}

}  // namespace

cudaError_t launch_bounded_wait(int32_t* status, unsigned long long timeout_ns, cudaStream_t s) {
  bounded_wait_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace calibatt
