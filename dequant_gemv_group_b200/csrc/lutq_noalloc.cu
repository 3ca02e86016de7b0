// lutq_gemv_noalloc: the fused GEMV with its scratch memory in a fixed,
// library-owned device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// product: code that records CUDA graphs in a capture mode where cudaMalloc
// is illegal, latency-critical serving loops that must not call cudaMalloc
// (it can block and synchronize the device), and plug-in hosts that give a
// library no allocator of its own.  This entry point lets them call the
// product with only their inputs and outputs.
//
// The scratch lives in g_noalloc_scratch below: a file-scope __device__ array
// of kNoallocScratchBytes (8 MiB).  Every GPU that loads the library holds
// that array until the process exits.  In host code the array's name is only a
// stand-in for a device symbol, so its device address is obtained once per
// device with cudaGetSymbolAddress, with that device current, on the first
// call made on that device.
//
// Layout: the first kNoallocZeroBytes (1 MiB) hold what the kernels need to
// find zero at the start of a call (exchange slots, arrival counters) and
// leave zero at its end; the partial sums that a call leaves behind go after
// them.  The same fixed split for every problem means no call's leftovers can
// land where a later call expects zeros, so the array is cleared once, at the
// set-up, and never again.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "lutq.h"
#include "lutq_trace.h"
#include "lutq_common.cuh"

namespace lutq {
cudaError_t launch_gemv(const void* x, int64_t M, const void* packed, const void* codebook,
                        int bits, int64_t N, int64_t K, float* y, void* workspace,
                        int32_t* dev_status, int num_sms, cudaStream_t stream,
                        bool y_bf16 = false, int64_t zero_bytes = -1, bool group64 = false);
int64_t gemm_scratch_bytes(int64_t M);
}  // namespace lutq

namespace {

constexpr int64_t kNoallocScratchBytes = int64_t(8) << 20;
constexpr int64_t kNoallocZeroBytes = int64_t(1) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch and multiprocessor count, per device.
// Written by the first call on a device; two host threads making that first
// call at once store the same values, so the race is harmless.
void* g_scratch_addr[kMaxDevices] = {nullptr};
int g_scratch_sms[kMaxDevices] = {0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" lutq_status lutq_gemv_noalloc(const void* x_bf16, int64_t M, const void* packed,
                                         const void* codebook_bf16, int bits, int64_t N,
                                         int64_t K, float* y, int32_t* dev_status,
                                         void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemv_noalloc");
  if (!x_bf16 || !packed || !codebook_bf16 || !y) return LUTQ_ERR_INVALID_ARG;
  if (bits != 3 && bits != 4) return LUTQ_ERR_BITS;
  if (N < lutq::kStrip || K < lutq::kGroup || N % lutq::kStrip != 0 || K % lutq::kGroup != 0 ||
      N > (int64_t(1) << 31) || K > (int64_t(1) << 31))
    return LUTQ_ERR_SHAPE;
  if (M < 1 || M > 16) return LUTQ_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(codebook_bf16) || !aligned16(y))
    return LUTQ_ERR_ALIGN;
  // The fixed array must hold this problem's scratch whichever kernel runs
  // it: its zero-at-start data in the first 1 MiB, its partial sums in the
  // rest.  Nothing is launched if not.
  const int64_t zero = lutq::workspace_zero_bytes(M, N, K);
  const int64_t scratch = lutq::gemm_scratch_bytes(M);
  if (zero > kNoallocZeroBytes || scratch > kNoallocScratchBytes - kNoallocZeroBytes)
    return LUTQ_ERR_WORKSPACE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LUTQ_ERR_CUDA;
  if (g_scratch_addr[dev] == nullptr) {
    // one-time set-up on this device (call it before any stream capture):
    // the array's address, the multiprocessor count, and the array cleared
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr)
      return LUTQ_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
      return LUTQ_ERR_CUDA;
    if (cudaMemset(addr, 0, size_t(kNoallocScratchBytes)) != cudaSuccess) return LUTQ_ERR_CUDA;
    g_scratch_sms[dev] = sms;
    g_scratch_addr[dev] = addr;
  }
  const cudaError_t err =
      lutq::launch_gemv(x_bf16, M, packed, codebook_bf16, bits, N, K, y, g_scratch_addr[dev],
                        dev_status, g_scratch_sms[dev], static_cast<cudaStream_t>(stream), false,
                        kNoallocZeroBytes);
  return err == cudaSuccess ? LUTQ_OK : LUTQ_ERR_CUDA;
}
