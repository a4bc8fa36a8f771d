// probe.cu — a kernel whose wait is never satisfied, for testing failure detection.
//
// One thread initialises an mbarrier that nothing ever arrives on and waits for its first phase
// with the library's bounded wait (mbar_wait, the helper every pipelined kernel uses). The wait
// runs out after kWaitLimitNs; the kernel records kDevWaitTimeout in the error word and returns.
// A stalled pipeline thus ends with a status the host reads (moe_check_error), and the context
// stays usable.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__global__ void __launch_bounds__(32) stalled_wait_kernel(int* err) {
  pdl_enter<false>();
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    // a fresh barrier is in phase 0, which completes only after one arrival: none comes
    if (!mbar_wait(smem_u32(&bar), 0u, nullptr)) flag_error(err, kDevWaitTimeout);
  }
}

}  // namespace

cudaError_t launch_stalled_wait(int* err, cudaStream_t stream) {
  return launch_kernel(stalled_wait_kernel, dim3(1), dim3(32), 0, stream, 1, err);
}

}  // namespace moe
