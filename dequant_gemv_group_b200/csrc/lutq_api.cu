// C ABI of liblutq: argument checks and kernel launches.  Every argument error
// is returned before anything is launched; device-side conditions go to the
// caller's dev_status word.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "lutq.h"
#include "lutq_trace.h"
#include "lutq_common.cuh"

namespace lutq {
cudaError_t launch_quantize(const void* W, int64_t N, int64_t K, const void* codebook, int bits,
                            uint8_t* codes, void* scales, int32_t* dev_status, int num_sms,
                            cudaStream_t stream, int scope = 0);
cudaError_t launch_pack(const uint8_t* codes, const void* scales, int64_t N, int64_t K,
                        int bits, void* packed, int32_t* dev_status, int num_sms,
                        cudaStream_t stream, bool group64 = false);
cudaError_t launch_gemv(const void* x, int64_t M, const void* packed, const void* codebook,
                        int bits, int64_t N, int64_t K, float* y, void* workspace,
                        int32_t* dev_status, int num_sms, cudaStream_t stream,
                        bool y_bf16 = false, int64_t zero_bytes = -1, bool group64 = false);
cudaError_t launch_gemm(const void* x, int64_t M, const void* packed, const void* codebook,
                        int bits, int64_t N, int64_t K, float* y, void* workspace,
                        int32_t* dev_status, int num_sms, cudaStream_t stream, int types = 0,
                        bool y_bf16 = false, int64_t zero_bytes = -1, bool group64 = false);
cudaError_t launch_gemv_rht(const void* x, int64_t M, const void* packed, const void* codebook,
                            const int8_t* signs, int bits, int64_t N, int64_t K, float* y,
                            void* workspace, int32_t* dev_status, int num_sms,
                            cudaStream_t stream);
bool gemv_small_path(int64_t M, int64_t K, int bits);
bool gemv_typed_path(int64_t M, int64_t K, int bits, int types);
cudaError_t launch_quantize_typed(const void* W, int64_t N, int64_t K, const void* codebooks,
                                  int types, int bits, uint8_t* codes, void* scales,
                                  uint8_t* group_types, int32_t* dev_status, int num_sms,
                                  cudaStream_t stream);
cudaError_t launch_pack_types(const uint8_t* types, int64_t N, int64_t K, int bits, void* packed,
                              int32_t* dev_status, int num_sms, cudaStream_t stream);
cudaError_t launch_gemv_typed(const void* x, int64_t M, const void* packed, const void* codebooks,
                              int types, int bits, int64_t N, int64_t K, float* y,
                              void* workspace, int32_t* dev_status, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_rht(const void* in, int64_t rows, int64_t K, const int8_t* signs,
                       bool activations, void* out, int num_sms, cudaStream_t stream);
cudaError_t launch_fit_histogram(const void* W, int64_t N, int64_t K, uint64_t* hist,
                                 int32_t* dev_status, int num_sms, cudaStream_t stream);
int64_t gemv_workspace_bytes(int64_t M, int64_t N);
void gemv_plan(int64_t N, int64_t K, int num_sms, int32_t* out);
int64_t gemm_counter_bytes(int64_t M, int64_t N);
int64_t gemm_scratch_bytes(int64_t M);

// The zero region of the workspace: the larger of the CUDA-core GEMV's
// exchange slots (M <= 4) and the tensor-core kernel's tile counters.  It
// does not depend on M up to M = 128 * 128 (the tensor-core kernel's
// counters grow with the number of 128-row batch tiles), so one workspace
// serves calls of any batch size up to the one it was sized for.
int64_t workspace_zero_bytes(int64_t M, int64_t N, int64_t K) {
  (void)K;
  const int64_t z = std::max(gemm_counter_bytes(M, N), gemv_workspace_bytes(4, N));
  return (z + 255) / 256 * 256;
}
}  // namespace lutq

namespace {

constexpr int kMaxDevices = 64;
int g_num_sms[kMaxDevices] = {0};

// Multiprocessor count of the current device (cached per device).
lutq_status current_sms(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LUTQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LUTQ_ERR_CUDA;
  if (g_num_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return LUTQ_ERR_CUDA;
    g_num_sms[dev] = n;
  }
  *out = g_num_sms[dev];
  return LUTQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lutq_status check_shape(int64_t N, int64_t K) {
  if (N < lutq::kStrip || K < lutq::kGroup) return LUTQ_ERR_SHAPE;
  if (N % lutq::kStrip != 0 || K % lutq::kGroup != 0) return LUTQ_ERR_SHAPE;
  if (N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return LUTQ_ERR_SHAPE;
  return LUTQ_OK;
}

lutq_status check_bits(int bits) { return (bits == 3 || bits == 4) ? LUTQ_OK : LUTQ_ERR_BITS; }

lutq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LUTQ_OK : LUTQ_ERR_CUDA; }

lutq_status check_product_args(const void* x, int64_t M, int64_t max_m, const void* packed,
                               const void* codebook, int bits, int64_t N, int64_t K,
                               const float* y, const void* workspace, int64_t workspace_bytes,
                               int64_t need) {
  if (!x || !packed || !codebook || !y) return LUTQ_ERR_INVALID_ARG;
  lutq_status st = check_bits(bits);
  if (st != LUTQ_OK) return st;
  st = check_shape(N, K);
  if (st != LUTQ_OK) return st;
  if (M < 1 || M > max_m) return LUTQ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(codebook) || !aligned16(y))
    return LUTQ_ERR_ALIGN;
  if (need > 0) {
    if (workspace == nullptr || workspace_bytes < need) return LUTQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return LUTQ_ERR_ALIGN;
  }
  return LUTQ_OK;
}

}  // namespace

extern "C" {

const char* lutq_status_string(int status) {
  LUTQ_TRACE_RANGE("lutq_status_string");
  switch (status) {
    case LUTQ_OK: return "LUTQ_OK";
    case LUTQ_ERR_INVALID_ARG: return "LUTQ_ERR_INVALID_ARG: null pointer or invalid value";
    case LUTQ_ERR_SHAPE: return "LUTQ_ERR_SHAPE: need N % 32 == 0, K % 128 == 0 and M in range";
    case LUTQ_ERR_BITS: return "LUTQ_ERR_BITS: bits must be 3 or 4 (and match the codebook)";
    case LUTQ_ERR_ALIGN: return "LUTQ_ERR_ALIGN: pointer not 16-byte aligned";
    case LUTQ_ERR_NONFINITE: return "LUTQ_ERR_NONFINITE: non-finite weight";
    case LUTQ_ERR_CODE_RANGE: return "LUTQ_ERR_CODE_RANGE: code >= 2^bits";
    case LUTQ_ERR_TIMEOUT: return "LUTQ_ERR_TIMEOUT: bounded wait expired inside a kernel";
    case LUTQ_ERR_CUDA: return "LUTQ_ERR_CUDA: CUDA runtime error";
    case LUTQ_ERR_WORKSPACE: return "LUTQ_ERR_WORKSPACE: workspace missing or too small";
    case LUTQ_ERR_BOUNDS: return "LUTQ_ERR_BOUNDS: an index outside its buffer (checked build)";
    default: return "unknown lutq status";
  }
}

int lutq_layout_version(void) {
  LUTQ_TRACE_RANGE("lutq_layout_version");
  return 2;
}

int lutq_build_flags(void) {
  LUTQ_TRACE_RANGE("lutq_build_flags");
  int flags = 0;
#ifdef LUTQ_NVTX
  flags |= LUTQ_BUILD_NVTX;
#endif
#ifdef LUTQ_BOUNDS
  flags |= LUTQ_BUILD_BOUNDS;
#endif
  return flags;
}

int64_t lutq_packed_bytes(int64_t N, int64_t K, int bits) {
  LUTQ_TRACE_RANGE("lutq_packed_bytes");
  if (check_shape(N, K) != LUTQ_OK || check_bits(bits) != LUTQ_OK) return -1;
  return (N / lutq::kStrip) * (K / lutq::kGroup) * (lutq::tile_bytes(bits) + lutq::kScaleBytes);
}

static lutq_status quantize(const void* W_bf16, int64_t N, int64_t K, const void* codebook_bf16,
                            int bits, uint8_t* codes, void* scales_bf16, int32_t* dev_status,
                            void* stream, int scope) {
  if (!W_bf16 || !codebook_bf16 || !codes || !scales_bf16) return LUTQ_ERR_INVALID_ARG;
  lutq_status st = check_bits(bits);
  if (st != LUTQ_OK) return st;
  if ((st = check_shape(N, K)) != LUTQ_OK) return st;
  if (scope == 3 && K % 256 != 0) return LUTQ_ERR_SHAPE;  // groups of 256
  if (!aligned16(W_bf16) || !aligned16(codebook_bf16) || !aligned16(codes) ||
      !aligned16(scales_bf16))
    return LUTQ_ERR_ALIGN;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_quantize(W_bf16, N, K, codebook_bf16, bits, codes, scales_bf16,
                                         dev_status, sms, static_cast<cudaStream_t>(stream),
                                         scope));
}

lutq_status lutq_quantize(const void* W_bf16, int64_t N, int64_t K, const void* codebook_bf16,
                          int bits, uint8_t* codes, void* scales_bf16, int32_t* dev_status,
                          void* stream) {
  LUTQ_TRACE_RANGE("lutq_quantize");
  return quantize(W_bf16, N, K, codebook_bf16, bits, codes, scales_bf16, dev_status, stream, 0);
}

lutq_status lutq_quantize_rowscale(const void* W_bf16, int64_t N, int64_t K,
                                   const void* codebook_bf16, int bits, uint8_t* codes,
                                   void* scales_bf16, int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_quantize_rowscale");
  return quantize(W_bf16, N, K, codebook_bf16, bits, codes, scales_bf16, dev_status, stream, 1);
}

lutq_status lutq_quantize_group256(const void* W_bf16, int64_t N, int64_t K,
                                   const void* codebook_bf16, int bits, uint8_t* codes,
                                   void* scales_bf16, int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_quantize_group256");
  return quantize(W_bf16, N, K, codebook_bf16, bits, codes, scales_bf16, dev_status, stream, 3);
}

lutq_status lutq_quantize_tensorscale(const void* W_bf16, int64_t N, int64_t K,
                                      const void* codebook_bf16, int bits, uint8_t* codes,
                                      void* scales_bf16, int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_quantize_tensorscale");
  return quantize(W_bf16, N, K, codebook_bf16, bits, codes, scales_bf16, dev_status, stream, 2);
}

lutq_status lutq_quantize_group64(const void* W_bf16, int64_t N, int64_t K,
                                  const void* codebook_bf16, int bits, uint8_t* codes,
                                  void* scales_bf16, int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_quantize_group64");
  return quantize(W_bf16, N, K, codebook_bf16, bits, codes, scales_bf16, dev_status, stream, 4);
}

static lutq_status pack(const uint8_t* codes, const void* scales_bf16, int64_t N, int64_t K,
                        int bits, void* packed, int32_t* dev_status, void* stream,
                        bool group64) {
  if (!codes || !scales_bf16 || !packed) return LUTQ_ERR_INVALID_ARG;
  lutq_status st = check_bits(bits);
  if (st != LUTQ_OK) return st;
  if ((st = check_shape(N, K)) != LUTQ_OK) return st;
  if (!aligned16(codes) || !aligned16(scales_bf16) || !aligned16(packed)) return LUTQ_ERR_ALIGN;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_pack(codes, scales_bf16, N, K, bits, packed, dev_status, sms,
                                     static_cast<cudaStream_t>(stream), group64));
}

lutq_status lutq_pack(const uint8_t* codes, const void* scales_bf16, int64_t N, int64_t K,
                      int bits, void* packed, int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_pack");
  return pack(codes, scales_bf16, N, K, bits, packed, dev_status, stream, false);
}

int64_t lutq_packed_bytes_group64(int64_t N, int64_t K, int bits) {
  LUTQ_TRACE_RANGE("lutq_packed_bytes_group64");
  if (check_shape(N, K) != LUTQ_OK || check_bits(bits) != LUTQ_OK) return -1;
  return (N / lutq::kStrip) * (K / lutq::kGroup) *
         (lutq::tile_bytes(bits) + 2 * lutq::kScaleBytes);
}

lutq_status lutq_pack_group64(const uint8_t* codes, const void* scales_bf16, int64_t N,
                              int64_t K, int bits, void* packed, int32_t* dev_status,
                              void* stream) {
  LUTQ_TRACE_RANGE("lutq_pack_group64");
  return pack(codes, scales_bf16, N, K, bits, packed, dev_status, stream, true);
}

lutq_status lutq_gemv_plan(int64_t N, int64_t K, int num_sms, int32_t* plan) {
  LUTQ_TRACE_RANGE("lutq_gemv_plan");
  if (plan == nullptr || num_sms < 1) return LUTQ_ERR_INVALID_ARG;
  lutq_status st;
  if ((st = check_shape(N, K)) != LUTQ_OK) return st;
  lutq::gemv_plan(N, K, num_sms, plan);
  return LUTQ_OK;
}

int64_t lutq_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  LUTQ_TRACE_RANGE("lutq_workspace_bytes");
  if (check_shape(N, K) != LUTQ_OK || check_bits(bits) != LUTQ_OK || M < 1) return -1;
  return lutq::workspace_zero_bytes(M, N, K) + lutq::gemm_scratch_bytes(M);
}

int64_t lutq_workspace_zero_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  LUTQ_TRACE_RANGE("lutq_workspace_zero_bytes");
  if (check_shape(N, K) != LUTQ_OK || check_bits(bits) != LUTQ_OK || M < 1) return -1;
  return lutq::workspace_zero_bytes(M, N, K);
}

lutq_status lutq_gemv(const void* x_bf16, int64_t M, const void* packed,
                      const void* codebook_bf16, int bits, int64_t N, int64_t K, float* y,
                      void* workspace, int64_t workspace_bytes, int32_t* dev_status,
                      void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemv");
  lutq_status st = check_product_args(x_bf16, M, 16, packed, codebook_bf16, bits, N, K, y,
                                      workspace, workspace_bytes,
                                      lutq_workspace_bytes(M, N, K, bits));
  if (st != LUTQ_OK) return st;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_gemv(x_bf16, M, packed, codebook_bf16, bits, N, K, y, workspace,
                                     dev_status, sms, static_cast<cudaStream_t>(stream)));
}

lutq_status lutq_gemv_out_bf16(const void* x_bf16, int64_t M, const void* packed,
                               const void* codebook_bf16, int bits, int64_t N, int64_t K,
                               void* y_bf16, void* workspace, int64_t workspace_bytes,
                               int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemv_out_bf16");
  lutq_status st = check_product_args(x_bf16, M, 16, packed, codebook_bf16, bits, N, K,
                                      static_cast<const float*>(y_bf16), workspace,
                                      workspace_bytes, lutq_workspace_bytes(M, N, K, bits));
  if (st != LUTQ_OK) return st;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_gemv(x_bf16, M, packed, codebook_bf16, bits, N, K,
                                     static_cast<float*>(y_bf16), workspace, dev_status, sms,
                                     static_cast<cudaStream_t>(stream), true));
}

lutq_status lutq_gemm_out_bf16(const void* x_bf16, int64_t M, const void* packed,
                               const void* codebook_bf16, int bits, int64_t N, int64_t K,
                               void* y_bf16, void* workspace, int64_t workspace_bytes,
                               int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemm_out_bf16");
  lutq_status st = check_product_args(x_bf16, M, int64_t(1) << 30, packed, codebook_bf16, bits,
                                      N, K, static_cast<const float*>(y_bf16), workspace,
                                      workspace_bytes, lutq_workspace_bytes(M, N, K, bits));
  if (st != LUTQ_OK) return st;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_gemm(x_bf16, M, packed, codebook_bf16, bits, N, K,
                                     static_cast<float*>(y_bf16), workspace, dev_status, sms,
                                     static_cast<cudaStream_t>(stream), 0, true));
}

lutq_status lutq_gemm(const void* x_bf16, int64_t M, const void* packed,
                      const void* codebook_bf16, int bits, int64_t N, int64_t K, float* y,
                      void* workspace, int64_t workspace_bytes, int32_t* dev_status,
                      void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemm");
  lutq_status st = check_product_args(x_bf16, M, int64_t(1) << 30, packed, codebook_bf16, bits,
                                      N, K, y, workspace, workspace_bytes,
                                      lutq_workspace_bytes(M, N, K, bits));
  if (st != LUTQ_OK) return st;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_gemm(x_bf16, M, packed, codebook_bf16, bits, N, K, y, workspace,
                                     dev_status, sms, static_cast<cudaStream_t>(stream)));
}

lutq_status lutq_gemv_group64(const void* x_bf16, int64_t M, const void* packed,
                              const void* codebook_bf16, int bits, int64_t N, int64_t K, float* y,
                              void* workspace, int64_t workspace_bytes, int32_t* dev_status,
                              void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemv_group64");
  lutq_status st = check_product_args(x_bf16, M, 16, packed, codebook_bf16, bits, N, K, y,
                                      workspace, workspace_bytes,
                                      lutq_workspace_bytes(M, N, K, bits));
  if (st != LUTQ_OK) return st;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_gemv(x_bf16, M, packed, codebook_bf16, bits, N, K, y, workspace,
                                     dev_status, sms, static_cast<cudaStream_t>(stream), false,
                                     -1, true));
}

lutq_status lutq_gemm_group64(const void* x_bf16, int64_t M, const void* packed,
                              const void* codebook_bf16, int bits, int64_t N, int64_t K, float* y,
                              void* workspace, int64_t workspace_bytes, int32_t* dev_status,
                              void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemm_group64");
  lutq_status st = check_product_args(x_bf16, M, int64_t(1) << 30, packed, codebook_bf16, bits,
                                      N, K, y, workspace, workspace_bytes,
                                      lutq_workspace_bytes(M, N, K, bits));
  if (st != LUTQ_OK) return st;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_gemm(x_bf16, M, packed, codebook_bf16, bits, N, K, y, workspace,
                                     dev_status, sms, static_cast<cudaStream_t>(stream), 0, false,
                                     -1, true));
}

static lutq_status rht(const void* in, int64_t rows, int64_t K, const int8_t* signs, void* out,
                       bool activations, void* stream) {
  if (!in || !signs || !out) return LUTQ_ERR_INVALID_ARG;
  if (rows < 1 || K < lutq::kGroup || K % lutq::kGroup != 0 || rows > (int64_t(1) << 31) ||
      K > (int64_t(1) << 31))
    return LUTQ_ERR_SHAPE;
  if (!aligned16(in) || !aligned16(signs) || !aligned16(out)) return LUTQ_ERR_ALIGN;
  const char* a = static_cast<const char*>(in);
  const char* b = static_cast<const char*>(out);
  const int64_t bytes = rows * K * 2;
  if (a < b + bytes && b < a + bytes) return LUTQ_ERR_INVALID_ARG;  // overlap
  int sms = 0;
  lutq_status st;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_rht(in, rows, K, signs, activations, out, sms,
                                    static_cast<cudaStream_t>(stream)));
}

lutq_status lutq_fit_histogram(const void* W_bf16, int64_t N, int64_t K, uint64_t* hist,
                               int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_fit_histogram");
  if (!W_bf16 || !hist) return LUTQ_ERR_INVALID_ARG;
  if (N < 1 || K < lutq::kGroup || K % lutq::kGroup != 0 || N > (int64_t(1) << 31) ||
      K > (int64_t(1) << 31))
    return LUTQ_ERR_SHAPE;
  if (!aligned16(W_bf16) || !aligned16(hist)) return LUTQ_ERR_ALIGN;
  int sms = 0;
  lutq_status st;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_fit_histogram(W_bf16, N, K, hist, dev_status, sms,
                                              static_cast<cudaStream_t>(stream)));
}

lutq_status lutq_rht_weights(const void* W_bf16, int64_t N, int64_t K, const int8_t* signs,
                             void* W_rot_bf16, void* stream) {
  LUTQ_TRACE_RANGE("lutq_rht_weights");
  return rht(W_bf16, N, K, signs, W_rot_bf16, false, stream);
}

lutq_status lutq_rht_activations(const void* x_bf16, int64_t M, int64_t K, const int8_t* signs,
                                 void* x_rot_bf16, void* stream) {
  LUTQ_TRACE_RANGE("lutq_rht_activations");
  return rht(x_bf16, M, K, signs, x_rot_bf16, true, stream);
}

lutq_status lutq_gemv_rht(const void* x_bf16, int64_t M, const void* packed,
                          const void* codebook_bf16, const int8_t* signs, int bits, int64_t N,
                          int64_t K, float* y, void* workspace, int64_t workspace_bytes,
                          int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemv_rht");
  if (!signs) return LUTQ_ERR_INVALID_ARG;
  lutq_status st = check_product_args(x_bf16, M, 16, packed, codebook_bf16, bits, N, K, y,
                                      workspace, workspace_bytes,
                                      lutq_workspace_bytes(M, N, K, bits));
  if (st != LUTQ_OK) return st;
  if (!aligned16(signs)) return LUTQ_ERR_ALIGN;
  if (!lutq::gemv_small_path(M, K, bits)) return LUTQ_ERR_SHAPE;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_gemv_rht(x_bf16, M, packed, codebook_bf16, signs, bits, N, K, y,
                                         workspace, dev_status, sms,
                                         static_cast<cudaStream_t>(stream)));
}

int lutq_max_types(int bits) {
  LUTQ_TRACE_RANGE("lutq_max_types");
  return check_bits(bits) == LUTQ_OK ? lutq::max_types(bits) : -1;
}

int64_t lutq_packed_bytes_typed(int64_t N, int64_t K, int bits) {
  LUTQ_TRACE_RANGE("lutq_packed_bytes_typed");
  const int64_t body = lutq_packed_bytes(N, K, bits);
  if (body < 0) return -1;
  return body + (N / lutq::kStrip) * (K / lutq::kGroup) * lutq::kTypeBytes;
}

lutq_status lutq_quantize_typed(const void* W_bf16, int64_t N, int64_t K,
                                const void* codebooks_bf16, int types, int bits, uint8_t* codes,
                                void* scales_bf16, uint8_t* group_types, int32_t* dev_status,
                                void* stream) {
  LUTQ_TRACE_RANGE("lutq_quantize_typed");
  if (!W_bf16 || !codebooks_bf16 || !codes || !scales_bf16 || !group_types)
    return LUTQ_ERR_INVALID_ARG;
  lutq_status st = check_bits(bits);
  if (st != LUTQ_OK) return st;
  if (types < 1 || types > lutq::max_types(bits)) return LUTQ_ERR_INVALID_ARG;
  if ((st = check_shape(N, K)) != LUTQ_OK) return st;
  if (!aligned16(W_bf16) || !aligned16(codebooks_bf16) || !aligned16(codes) ||
      !aligned16(scales_bf16) || !aligned16(group_types))
    return LUTQ_ERR_ALIGN;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_quantize_typed(W_bf16, N, K, codebooks_bf16, types, bits, codes,
                                               scales_bf16, group_types, dev_status, sms,
                                               static_cast<cudaStream_t>(stream)));
}

lutq_status lutq_pack_typed(const uint8_t* codes, const void* scales_bf16,
                            const uint8_t* group_types, int64_t N, int64_t K, int bits,
                            void* packed, int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_pack_typed");
  if (!group_types) return LUTQ_ERR_INVALID_ARG;
  if (!aligned16(group_types)) return LUTQ_ERR_ALIGN;
  lutq_status st = lutq_pack(codes, scales_bf16, N, K, bits, packed, dev_status, stream);
  if (st != LUTQ_OK) return st;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_pack_types(group_types, N, K, bits, packed, dev_status, sms,
                                           static_cast<cudaStream_t>(stream)));
}

lutq_status lutq_gemv_typed(const void* x_bf16, int64_t M, const void* packed,
                            const void* codebooks_bf16, int types, int bits, int64_t N, int64_t K,
                            float* y, void* workspace, int64_t workspace_bytes,
                            int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemv_typed");
  lutq_status st = check_product_args(x_bf16, M, 16, packed, codebooks_bf16, bits, N, K, y,
                                      workspace, workspace_bytes,
                                      lutq_workspace_bytes(M, N, K, bits));
  if (st != LUTQ_OK) return st;
  if (types < 1 || types > lutq::max_types(bits)) return LUTQ_ERR_INVALID_ARG;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_gemv_typed(x_bf16, M, packed, codebooks_bf16, types, bits, N, K,
                                           y, workspace, dev_status, sms,
                                           static_cast<cudaStream_t>(stream)));
}

lutq_status lutq_gemm_typed(const void* x_bf16, int64_t M, const void* packed,
                            const void* codebooks_bf16, int types, int bits, int64_t N, int64_t K,
                            float* y, void* workspace, int64_t workspace_bytes,
                            int32_t* dev_status, void* stream) {
  LUTQ_TRACE_RANGE("lutq_gemm_typed");
  lutq_status st = check_product_args(x_bf16, M, int64_t(1) << 30, packed, codebooks_bf16, bits,
                                      N, K, y, workspace, workspace_bytes,
                                      lutq_workspace_bytes(M, N, K, bits));
  if (st != LUTQ_OK) return st;
  if (types < 1 || types > lutq::max_types(bits)) return LUTQ_ERR_INVALID_ARG;
  int sms = 0;
  if ((st = current_sms(&sms)) != LUTQ_OK) return st;
  return from_cuda(lutq::launch_gemm(x_bf16, M, packed, codebooks_bf16, bits, N, K, y, workspace,
                                     dev_status, sms, static_cast<cudaStream_t>(stream), types));
}

}  // extern "C"
