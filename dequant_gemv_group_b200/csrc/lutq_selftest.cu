// lutq_selftest_wait_timeout: runs the bounded mbarrier wait that every
// pipeline wait of the GEMV and GEMM kernels uses, on a barrier that nothing
// completes, so that a caller (or a test) can see the time limit end the wait,
// the kernel report LUTQ_ERR_TIMEOUT and the context stay usable.
#include <cstdint>
#include <cuda_runtime.h>

#include "lutq.h"
#include "lutq_common.cuh"
#include "lutq_sm100.cuh"

namespace {

__global__ void wait_timeout_kernel(int32_t* dev_status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  const uint32_t b = lutq::sm100::smem_addr(&bar);
  lutq::sm100::mbar_init(b, 1);  // one arrival expected; none comes
  lutq::sm100::mbar_fence_init();
  if (!lutq::sm100::mbar_wait(b, 0, &abort_flag, limit_ns))
    lutq::report(dev_status, LUTQ_ERR_TIMEOUT);
}

}  // namespace

extern "C" lutq_status lutq_selftest_wait_timeout(int32_t* dev_status, int64_t limit_ns,
                                                  void* stream) {
  if (dev_status == nullptr || limit_ns < 1 || limit_ns > 1000000000) return LUTQ_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status,
                                                                       uint64_t(limit_ns));
  return cudaGetLastError() == cudaSuccess ? LUTQ_OK : LUTQ_ERR_CUDA;
}
