// Self-test of the bounded-wait machinery used by the tensor-core kernels:
// a kernel waits on an mbarrier that nothing ever arrives at and must give up
// after the wait limit with MOBA_ERR_TIMEOUT in the status word, leaving the
// context usable.  Nothing faults, traps or hangs.
#include "launch.h"
#include "sm100.cuh"

namespace moba {

namespace {

__global__ void bounded_wait_selftest_kernel(int* status) {
  __shared__ uint64_t never_arrived;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&never_arrived);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = sm100::mbar_wait(b, 0, &abort_flag);
    *status = ok ? (int)MOBA_OK : (abort_flag ? (int)MOBA_ERR_TIMEOUT : (int)MOBA_ERR_INTERNAL);
  }
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int* status, cudaStream_t stream) {
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace moba
