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
// The scratch (the exchange slots where lutq_gemv meets the two halves of a
// strip split between two CTAs) lives in g_noalloc_scratch below: a file-scope
// __device__ array of kNoallocScratchBytes (4 MiB).  Every GPU that loads the
// library holds that array until the process exits.  In host code the
// array's name is only a stand-in for a device symbol, so its device address
// is obtained once per device with cudaGetSymbolAddress, with that device
// current, on the first call made on that device.
#include <cstdint>
#include <cuda_runtime.h>

#include "lutq.h"
#include "lutq_common.cuh"

namespace lutq {
cudaError_t launch_gemv(const void* x, int64_t M, const void* packed, const void* codebook,
                        int bits, int64_t N, int64_t K, float* y, void* workspace,
                        int32_t* dev_status, int num_sms, cudaStream_t stream,
                        bool y_bf16 = false);
int64_t gemv_workspace_bytes(int64_t M, int64_t N);
}  // namespace lutq

namespace {

constexpr int64_t kNoallocScratchBytes = int64_t(4) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch and multiprocessor count, per device.
void* g_scratch_addr[kMaxDevices] = {nullptr};
int g_scratch_sms[kMaxDevices] = {0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" lutq_status lutq_gemv_noalloc(const void* x_bf16, int64_t M, const void* packed,
                                         const void* codebook_bf16, int bits, int64_t N,
                                         int64_t K, float* y, int32_t* dev_status,
                                         void* stream) {
  if (!x_bf16 || !packed || !codebook_bf16 || !y) return LUTQ_ERR_INVALID_ARG;
  if (bits != 3 && bits != 4) return LUTQ_ERR_BITS;
  if (N < lutq::kStrip || K < lutq::kGroup || N % lutq::kStrip != 0 || K % lutq::kGroup != 0 ||
      N > (int64_t(1) << 31) || K > (int64_t(1) << 31))
    return LUTQ_ERR_SHAPE;
  if (M < 1 || M > 16) return LUTQ_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(codebook_bf16) || !aligned16(y))
    return LUTQ_ERR_ALIGN;
  // The fixed array must hold this problem's scratch; nothing is launched if not.
  const int64_t need = lutq::gemv_workspace_bytes(M, N);
  if (need > kNoallocScratchBytes) return LUTQ_ERR_WORKSPACE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LUTQ_ERR_CUDA;
  if (g_scratch_addr[dev] == nullptr) {
    // one-time set-up on this device (call it before any stream capture)
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr)
      return LUTQ_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
      return LUTQ_ERR_CUDA;
    g_scratch_sms[dev] = sms;
    g_scratch_addr[dev] = addr;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents; the exchange slots this
  // problem uses must begin at zero.
  if (cudaMemsetAsync(g_scratch_addr[dev], 0, size_t(need), s) != cudaSuccess)
    return LUTQ_ERR_CUDA;
  const cudaError_t err =
      lutq::launch_gemv(x_bf16, M, packed, codebook_bf16, bits, N, K, y, g_scratch_addr[dev],
                        dev_status, g_scratch_sms[dev], s);
  return err == cudaSuccess ? LUTQ_OK : LUTQ_ERR_CUDA;
}
