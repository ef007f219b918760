// selftest.cu -- the bounded wait, exercised on purpose.
//
// Every wait of the library's kernels on an mbarrier gives up after kWaitLimitNs, records
// MOE_ERR_DEVICE_TIMEOUT in the workspace's status word and lets the kernel return, so a
// stalled pipeline ends with an error the host reads instead of a hang.  This kernel runs
// that same wait on a barrier that nothing ever completes.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "moe_layer.h"

namespace moe {

__global__ void wait_timeout_kernel(Ctrl* ctrl) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none ever comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && mbar_wait(&bar, 0, ctrl, &abort_flag)) set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
}

}  // namespace moe

extern "C" moe_status moe_layer_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                                      void* stream) {
  if (!workspace || workspace_bytes < sizeof(moe::Ctrl) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  moe::Ctrl* ctrl = static_cast<moe::Ctrl*>(workspace);
  if (cudaMemsetAsync(ctrl, 0, sizeof(moe::Ctrl), st) != cudaSuccess) return MOE_ERR_CUDA;
  moe::wait_timeout_kernel<<<1, 32, 0, st>>>(ctrl);
  moe::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
