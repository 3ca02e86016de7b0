// Histogram of a layer's normalised weights, the data of a codebook fitted to
// the layer (Lloyd-Max on the layer's own weights: "TurboQuant: A
// first-principles walkthrough" names the algorithm).  Each weight's
// v = fp32(w) / fp32(s), s the absolute maximum of its group of 128 (the value
// lutq_quantize compares with the levels), falls in bin
// floor(fp32(v + 1) * kHistBins / 2), clamped to the last bin.  One warp per
// group (four weights a lane); counts go to a shared-memory histogram per
// block and then, once per block, to the caller's 64-bit counters.
#include "lutq_common.cuh"

namespace lutq {

constexpr int kHistBins = 16384;

__global__ void __launch_bounds__(512) fit_hist_kernel(const uint16_t* __restrict__ W, int64_t N,
                                                       int64_t K, unsigned long long* hist,
                                                       int32_t* dev_status) {
  extern __shared__ uint32_t sh[];  // [kHistBins]
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t groups = N * (K / kGroup);
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  bool bad = false;
  for (int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < groups;
       t += warps) {
    const uint2 raw = *reinterpret_cast<const uint2*>(W + t * kGroup + 4 * lane);
    const float w[4] = {bf16_lo_to_f32(raw.x), bf16_hi_to_f32(raw.x), bf16_lo_to_f32(raw.y),
                        bf16_hi_to_f32(raw.y)};
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      bad |= !isfinite(w[i]);
      m = fmaxf(m, fabsf(w[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // the quantizer's IEEE divide; then v + 1 rounded on its own before the
      // (exact) scaling by a power of two
      const float v = m > 0.0f ? __fdiv_rn(w[i], m) : 0.0f;
      int b = int(floorf(__fmul_rn(__fadd_rn(v, 1.0f), float(kHistBins / 2))));
      b = b < 0 ? 0 : (b >= kHistBins ? kHistBins - 1 : b);
      atomicAdd(&sh[b], 1u);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(dev_status, LUTQ_ERR_NONFINITE);
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (sh[i] != 0) atomicAdd(&hist[i], static_cast<unsigned long long>(sh[i]));
}

cudaError_t launch_fit_histogram(const void* W, int64_t N, int64_t K, uint64_t* hist,
                                 int32_t* dev_status, int num_sms, cudaStream_t stream) {
  constexpr int kSmem = kHistBins * 4;
  const cudaError_t e =
      cudaFuncSetAttribute(fit_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const int64_t groups = N * (K / kGroup);
  int64_t blocks = (groups + 15) / 16;
  if (blocks > int64_t(num_sms) * 2) blocks = int64_t(num_sms) * 2;
  if (blocks < 1) blocks = 1;
  fit_hist_kernel<<<unsigned(blocks), 512, kSmem, stream>>>(
      static_cast<const uint16_t*>(W), N, K, reinterpret_cast<unsigned long long*>(hist),
      dev_status);
  return cudaGetLastError();
}

}  // namespace lutq
