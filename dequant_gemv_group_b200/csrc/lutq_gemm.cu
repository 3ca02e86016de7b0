// Tensor-core (tcgen05) dequantize-and-multiply for batches that form a dense
// contraction.  Not built yet: the entry point reports a CUDA error.
#include "lutq_common.cuh"

namespace lutq {

int64_t gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

cudaError_t launch_gemm(const void*, int64_t, const void*, const void*, const void*, int, int64_t,
                        int64_t, float*, void*, int32_t*, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace lutq
