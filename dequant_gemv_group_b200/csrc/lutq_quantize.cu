// Group-128 round-to-nearest quantization onto a codebook (the RTN step of the
// group-128 post-training-quantization study and the FLUTE abstract, "Daily
// Papers" listing, query "group-128").
//
// One warp handles one (row, group) unit at a time: each lane loads 4 of the
// group's 128 bf16 weights (8 bytes), the warp reduces |w| to the group's
// absolute maximum s, and every lane maps its 4 weights to the lowest index
// minimising the fp32 distance |w/s - c_i|.  This translation unit is built
// without fused multiply-add contraction or flush-to-zero, and the divide is
// the IEEE round-to-nearest division.
#include "lutq_common.cuh"

namespace lutq {

template <int BITS>
__global__ void __launch_bounds__(256)
quantize_kernel(const uint2* __restrict__ W, int64_t n_rows, int64_t groups,
                const uint16_t* __restrict__ codebook, uint32_t* __restrict__ codes,
                uint16_t* __restrict__ scales, int32_t* dev_status) {
  constexpr int L = 1 << BITS;
  __shared__ float levels[L];
  if (threadIdx.x < L) levels[threadIdx.x] = __uint_as_float(uint32_t(codebook[threadIdx.x]) << 16);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const int64_t units = n_rows * groups;
  bool bad = false;
  for (int64_t u = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units;
       u += warps) {
    // unit u = (row, group) in row-major order; 32 lanes x 4 weights = 128
    const uint2 raw = W[u * 32 + lane];
    float w[4] = {bf16_lo_to_f32(raw.x), bf16_hi_to_f32(raw.x),
                  bf16_lo_to_f32(raw.y), bf16_hi_to_f32(raw.y)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (!isfinite(w[i])) bad = true;
      amax = fmaxf(amax, fabsf(w[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));

    uint32_t packed4 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float v = amax > 0.0f ? __fdiv_rn(w[i], amax) : 0.0f;
      float best = INFINITY;
      uint32_t bi = 0;
#pragma unroll
      for (int c = 0; c < L; ++c) {
        const float d = fabsf(__fsub_rn(v, levels[c]));
        if (d < best) { best = d; bi = c; }
      }
      packed4 |= bi << (8 * i);
    }
    codes[u * 32 + lane] = packed4;
    if (lane == 0) scales[u] = uint16_t(__float_as_uint(amax) >> 16);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(dev_status, LUTQ_ERR_NONFINITE);
}

cudaError_t launch_quantize(const void* W, int64_t N, int64_t K, const void* codebook, int bits,
                            uint8_t* codes, void* scales, int32_t* dev_status, int num_sms,
                            cudaStream_t stream) {
  const int64_t units = N * (K / kGroup);
  int64_t blocks = (units + 7) / 8;
  const int64_t cap = int64_t(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (bits == 4)
    quantize_kernel<4><<<unsigned(blocks), 256, 0, stream>>>(
        static_cast<const uint2*>(W), N, K / kGroup, static_cast<const uint16_t*>(codebook),
        reinterpret_cast<uint32_t*>(codes), static_cast<uint16_t*>(scales), dev_status);
  else
    quantize_kernel<3><<<unsigned(blocks), 256, 0, stream>>>(
        static_cast<const uint2*>(W), N, K / kGroup, static_cast<const uint16_t*>(codebook),
        reinterpret_cast<uint32_t*>(codes), static_cast<uint16_t*>(scales), dev_status);
  return cudaGetLastError();
}

}  // namespace lutq
