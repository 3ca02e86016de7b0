// lutq_selftest_wait_timeout: runs the bounded mbarrier wait that every
// pipeline wait of the GEMV and GEMM kernels uses, on a barrier that nothing
// completes, so that a caller (or a test) can see the time limit end the wait,
// the kernel report LUTQ_ERR_TIMEOUT and the context stay usable.
// lutq_selftest_bounds: runs the kernels' index check on an index one past
// the extent it is given, inside a larger array, so that a checked build can
// be seen to report LUTQ_ERR_BOUNDS and skip the access.
#include <cstdint>
#include <cuda_runtime.h>

#include "lutq.h"
#include "lutq_trace.h"
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

// Writes element `idx` of a 64-element shared array through the index check
// with extent 32: idx = 32 is past the extent but inside the array.
__global__ void bounds_kernel(int32_t* dev_status, int idx) {
  __shared__ int buf[64];
  if (threadIdx.x != 0) return;
  if (idx < 0 || idx >= 64) return;
  buf[0] = 0;
  if (LUTQ_IN_BOUNDS(idx < 32, dev_status)) buf[idx] = 1;
  if (buf[0] != 0) lutq::report(dev_status, LUTQ_ERR_INVALID_ARG);  // only idx = 0 writes it
}

}  // namespace

extern "C" lutq_status lutq_selftest_bounds(int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_selftest_bounds");
  if (dev_status == nullptr) return LUTQ_ERR_INVALID_ARG;
  bounds_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status, 32);
  return cudaGetLastError() == cudaSuccess ? LUTQ_OK : LUTQ_ERR_CUDA;
}

extern "C" lutq_status lutq_selftest_wait_timeout(int32_t* dev_status, int64_t limit_ns,
                                                  void* stream) {
  LUTQ_TRACE_RANGE("lutq_selftest_wait_timeout");
  if (dev_status == nullptr || limit_ns < 1 || limit_ns > 1000000000) return LUTQ_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status,
                                                                       uint64_t(limit_ns));
  return cudaGetLastError() == cudaSuccess ? LUTQ_OK : LUTQ_ERR_CUDA;
}
