// Randomized Hadamard rotation of weights (offline) and activations (for
// lutq_gemm, or any other consumer): every 128-long group of a row becomes
// H diag(s) g (weights, summed in fp64) or H diag(s) g / 128 (activations,
// summed in fp32, the arithmetic of the fused GEMV), rounded once to bf16
// ("TurboQuant: A first-principles walkthrough": randomized Hadamard
// transforms can replace uniform random rotations).  One warp per (row,
// group), grid-stride.
#include <cuda_bf16.h>

#include "lutq_common.cuh"
#include "lutq_rht.cuh"

namespace lutq {

__device__ __forceinline__ uint32_t to_bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
__device__ __forceinline__ uint32_t to_bf16_bits(double v) {
  return __bfloat16_as_ushort(__double2bfloat16(v));
}

// Weights: one warp per (row, group) task, butterflies in T = double;
// post_scale 1.
template <typename T>
__global__ void __launch_bounds__(256) rht_kernel(const uint16_t* __restrict__ in, int64_t rows,
                                                  int64_t K, const int8_t* __restrict__ signs,
                                                  T post_scale, uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const uint32_t signs4 = reinterpret_cast<const uint32_t*>(signs)[lane];
  const int64_t G = K / kGroup;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < rows * G;
       t += warps) {
    const int64_t off = t * kGroup + 4 * lane;  // row-major: group t of all rows in order
    const uint2 raw = *reinterpret_cast<const uint2*>(in + off);
    T v[4] = {T(bf16_lo_to_f32(raw.x)), T(bf16_hi_to_f32(raw.x)), T(bf16_lo_to_f32(raw.y)),
              T(bf16_hi_to_f32(raw.y))};
    rht128_warp(v, signs4);
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = to_bf16_bits(v[i] * post_scale);
    *reinterpret_cast<uint2*>(out + off) = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
  }
}

// Activations: eight lanes per (row, group) task, four tasks per warp, the
// arithmetic of the fused GEMV prologue.
__global__ void __launch_bounds__(256) rht_act_kernel(const uint16_t* __restrict__ in,
                                                      int64_t rows, int64_t K,
                                                      const int8_t* __restrict__ signs,
                                                      uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const uint4 signs16 = reinterpret_cast<const uint4*>(signs)[lane & 7];
  const int64_t tasks = rows * (K / kGroup);
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t0 = 4 * (int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5));
       t0 < tasks; t0 += 4 * warps) {
    const int64_t t = t0 + (lane >> 3);
    const int64_t off = t * kGroup + 16 * (lane & 7);
    uint4 r0 = make_uint4(0, 0, 0, 0), r1 = r0;
    if (t < tasks) {
      r0 = *reinterpret_cast<const uint4*>(in + off);
      r1 = *reinterpret_cast<const uint4*>(in + off + 8);
    }
    const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = bf16_lo_to_f32(w[i]);
      v[2 * i + 1] = bf16_hi_to_f32(w[i]);
    }
    rht128_octet(v, signs16);
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      h[i] = to_bf16_bits(v[2 * i] * (1.0f / kGroup)) |
             (to_bf16_bits(v[2 * i + 1] * (1.0f / kGroup)) << 16);
    if (t < tasks) {
      *reinterpret_cast<uint4*>(out + off) = make_uint4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<uint4*>(out + off + 8) = make_uint4(h[4], h[5], h[6], h[7]);
    }
  }
}

cudaError_t launch_rht(const void* in, int64_t rows, int64_t K, const int8_t* signs,
                       bool activations, void* out, int num_sms, cudaStream_t stream) {
  const int64_t tasks = rows * (K / kGroup);
  int64_t blocks = (tasks + 7) / 8;
  if (blocks > int64_t(num_sms) * 16) blocks = int64_t(num_sms) * 16;
  if (blocks < 1) blocks = 1;
  const uint16_t* src = static_cast<const uint16_t*>(in);
  uint16_t* dst = static_cast<uint16_t*>(out);
  if (activations)
    rht_act_kernel<<<unsigned(blocks), 256, 0, stream>>>(src, rows, K, signs, dst);
  else
    rht_kernel<double><<<unsigned(blocks), 256, 0, stream>>>(src, rows, K, signs, 1.0, dst);
  return cudaGetLastError();
}

}  // namespace lutq
