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

// SCOPE of the scale: 0, the group's absolute maximum; 1, one scale per row
// (Tetra abstract, aiqbench news item: one scale per matrix row; here the
// row's absolute maximum), which row_amax_kernel has left in the row's first
// scale slot; 2, one scale for the matrix (the tensor-wise granularity of the
// Log_bQuant abstract's baseline), left in the first slot of row 0 by
// tensor_amax_kernel; 3, one scale per group of 256 along K (the group-size
// variant), left in the even 128-group's slot by pair_amax_kernel; 4, one
// scale per group of 64 (the finer group-size variant): the two half-warps
// reduce their own 64 weights and write scales [N, K/64], slot 2 u + half.
// Every group divides by its scale; with scopes 1-3 the other slots receive a
// copy.
template <int BITS, int SCOPE>
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
    for (int off = SCOPE == 4 ? 8 : 16; off > 0; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const int64_t g = u % groups;
    if (SCOPE == 1) amax = __uint_as_float(uint32_t(scales[u - g]) << 16);
    if (SCOPE == 2) amax = __uint_as_float(uint32_t(scales[0]) << 16);
    if (SCOPE == 3) amax = __uint_as_float(uint32_t(scales[u - (g & 1)]) << 16);

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
    const bool source =
        (SCOPE == 1 && g == 0) || (SCOPE == 2 && u == 0) || (SCOPE == 3 && (g & 1) == 0);
    if (SCOPE == 4) {
      if ((lane & 15) == 0) scales[2 * u + (lane >> 4)] = uint16_t(__float_as_uint(amax) >> 16);
    } else if (lane == 0 && !source) {
      scales[u] = uint16_t(__float_as_uint(amax) >> 16);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(dev_status, LUTQ_ERR_NONFINITE);
}

// The absolute maximum of each row (one warp per row, 16-byte loads), as
// bf16 bits (exact: the maximum of bf16 magnitudes) into the row's first
// scale slot.
__global__ void __launch_bounds__(256)
row_amax_kernel(const uint4* __restrict__ W, int64_t n_rows, int64_t K, int64_t groups,
                uint16_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n_rows;
       r += warps) {
    const uint4* row = W + r * (K / 8);
    float amax = 0.0f;
    for (int64_t j = lane; j < K / 8; j += 32) {
      const uint4 v = row[j];
      const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_lo_to_f32(x[i])), fabsf(bf16_hi_to_f32(x[i]))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) scales[r * groups] = uint16_t(__float_as_uint(amax) >> 16);
  }
}

// Per-group data types (BitMoD abstract, same listing: each group of 128
// weights may be quantized with its own data type).  One thread per (row,
// group): the absolute maximum, then for every type t the RTN codes and the
// squared error E_t = sum over k = 0..127, in that order, of d * d in fp64,
// d = fp32(v - c_t[q]) the RTN distance (each product exact, each addition
// rounded once); the group takes the lowest t of smallest E_t and is written
// with that type's codes.  codebooks: [types][2^BITS] bf16.
template <int BITS>
__global__ void __launch_bounds__(256)
quantize_typed_kernel(const uint4* __restrict__ W, int64_t units,
                      const uint16_t* __restrict__ codebooks, int types,
                      uint2* __restrict__ codes, uint16_t* __restrict__ scales,
                      uint8_t* __restrict__ group_types, int32_t* dev_status) {
  constexpr int L = 1 << BITS;
  constexpr int kMaxTypes = 4;
  __shared__ float levels[kMaxTypes][L];
  for (int i = threadIdx.x; i < types * L; i += blockDim.x)
    levels[i / L][i % L] = __uint_as_float(uint32_t(codebooks[i]) << 16);
  __syncthreads();

  // the lowest index of smallest fp32 distance |v - c_i| (as quantize_kernel)
  auto nearest = [&](float v, int t) -> uint32_t {
    float best = INFINITY;
    uint32_t bi = 0;
#pragma unroll
    for (int c = 0; c < L; ++c) {
      const float d = fabsf(__fsub_rn(v, levels[t][c]));
      if (d < best) {
        best = d;
        bi = c;
      }
    }
    return bi;
  };
  auto values = [](const uint4& r, float (&w)[8]) {
    const uint32_t x[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      w[2 * i] = bf16_lo_to_f32(x[i]);
      w[2 * i + 1] = bf16_hi_to_f32(x[i]);
    }
  };

  bool bad = false;
  for (int64_t u = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; u < units;
       u += int64_t(gridDim.x) * blockDim.x) {
    const uint4* src = W + u * (kGroup / 8);
    float amax = 0.0f;
    for (int j = 0; j < kGroup / 8; ++j) {
      float w[8];
      values(src[j], w);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (!isfinite(w[i])) bad = true;
        amax = fmaxf(amax, fabsf(w[i]));
      }
    }
    double err[kMaxTypes] = {0.0, 0.0, 0.0, 0.0};
    for (int j = 0; j < kGroup / 8; ++j) {
      float w[8];
      values(src[j], w);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v = amax > 0.0f ? __fdiv_rn(w[i], amax) : 0.0f;
#pragma unroll
        for (int t = 0; t < kMaxTypes; ++t) {
          if (t >= types) break;
          const double d = double(__fsub_rn(v, levels[t][nearest(v, t)]));
          err[t] = __dadd_rn(err[t], __dmul_rn(d, d));
        }
      }
    }
    int pick = 0;
    double best = err[0];
#pragma unroll
    for (int t = 1; t < kMaxTypes; ++t)
      if (t < types && err[t] < best) {
        best = err[t];
        pick = t;
      }
    for (int j = 0; j < kGroup / 8; ++j) {
      float w[8];
      values(src[j], w);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v = amax > 0.0f ? __fdiv_rn(w[i], amax) : 0.0f;
        const uint32_t q = nearest(v, pick);
        if (i < 4)
          lo |= q << (8 * i);
        else
          hi |= q << (8 * (i - 4));
      }
      codes[u * (kGroup / 8) + j] = make_uint2(lo, hi);
    }
    scales[u] = uint16_t(__float_as_uint(amax) >> 16);
    group_types[u] = uint8_t(pick);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) report(dev_status, LUTQ_ERR_NONFINITE);
}

cudaError_t launch_quantize_typed(const void* W, int64_t N, int64_t K, const void* codebooks,
                                  int types, int bits, uint8_t* codes, void* scales,
                                  uint8_t* group_types, int32_t* dev_status, int num_sms,
                                  cudaStream_t stream) {
  const int64_t units = N * (K / kGroup);
  int64_t blocks = (units + 255) / 256;
  const int64_t cap = int64_t(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const uint4* w = static_cast<const uint4*>(W);
  const uint16_t* cb = static_cast<const uint16_t*>(codebooks);
  uint2* c = reinterpret_cast<uint2*>(codes);
  uint16_t* s = static_cast<uint16_t*>(scales);
  if (bits == 4)
    quantize_typed_kernel<4><<<unsigned(blocks), 256, 0, stream>>>(w, units, cb, types, c, s,
                                                                    group_types, dev_status);
  else
    quantize_typed_kernel<3><<<unsigned(blocks), 256, 0, stream>>>(w, units, cb, types, c, s,
                                                                    group_types, dev_status);
  return cudaGetLastError();
}

// The absolute maximum of each group of 256 along K (one warp per group, one
// 16-byte load per lane) as bf16 bits into the slot of its even 128-group.
// groups (of 128) is even.
__global__ void __launch_bounds__(256)
pair_amax_kernel(const uint4* __restrict__ W, int64_t n_rows, int64_t K, int64_t groups,
                 uint16_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t pairs = groups / 2;
  const int64_t tasks = n_rows * pairs;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < tasks;
       t += warps) {
    const int64_t row = t / pairs, j = t - row * pairs;
    const uint4 v = W[row * (K / 8) + j * 32 + lane];
    const uint32_t x[4] = {v.x, v.y, v.z, v.w};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      amax = fmaxf(amax, fmaxf(fabsf(bf16_lo_to_f32(x[i])), fabsf(bf16_hi_to_f32(x[i]))));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) scales[row * groups + 2 * j] = uint16_t(__float_as_uint(amax) >> 16);
  }
}

// The maximum of the rows' maxima (left by row_amax_kernel in each row's
// first slot) into the first slot of row 0: one block.
__global__ void __launch_bounds__(1024)
tensor_amax_kernel(int64_t n_rows, int64_t groups, uint16_t* __restrict__ scales) {
  __shared__ uint32_t best;
  if (threadIdx.x == 0) best = 0;
  __syncthreads();
  uint32_t m = 0;  // bf16 bits of non-negative values order as integers
  for (int64_t r = threadIdx.x; r < n_rows; r += blockDim.x) m = max(m, uint32_t(scales[r * groups]));
  atomicMax(&best, m);
  __syncthreads();
  if (threadIdx.x == 0) scales[0] = uint16_t(best);
}

cudaError_t launch_quantize(const void* W, int64_t N, int64_t K, const void* codebook, int bits,
                            uint8_t* codes, void* scales, int32_t* dev_status, int num_sms,
                            cudaStream_t stream, int scope) {
  const int64_t units = N * (K / kGroup);
  int64_t blocks = (units + 7) / 8;
  const int64_t cap = int64_t(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  const uint2* w = static_cast<const uint2*>(W);
  const uint16_t* cb = static_cast<const uint16_t*>(codebook);
  uint32_t* c = reinterpret_cast<uint32_t*>(codes);
  uint16_t* s = static_cast<uint16_t*>(scales);
  if (scope == 3) {
    int64_t pb = (N * (K / 256) + 7) / 8;
    if (pb > int64_t(num_sms) * 16) pb = int64_t(num_sms) * 16;
    pair_amax_kernel<<<unsigned(pb), 256, 0, stream>>>(static_cast<const uint4*>(W), N, K,
                                                       K / kGroup, s);
  }
  if (scope == 1 || scope == 2) {
    int64_t rb = (N + 7) / 8;
    if (rb > int64_t(num_sms) * 8) rb = int64_t(num_sms) * 8;
    row_amax_kernel<<<unsigned(rb), 256, 0, stream>>>(static_cast<const uint4*>(W), N, K,
                                                      K / kGroup, s);
  }
  if (scope == 2) tensor_amax_kernel<<<1, 1024, 0, stream>>>(N, K / kGroup, s);
  const int64_t G = K / kGroup;
  switch (scope * 2 + (bits == 4 ? 1 : 0)) {
    case 0: quantize_kernel<3, 0><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
    case 1: quantize_kernel<4, 0><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
    case 2: quantize_kernel<3, 1><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
    case 3: quantize_kernel<4, 1><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
    case 4: quantize_kernel<3, 2><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
    case 5: quantize_kernel<4, 2><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
    case 6: quantize_kernel<3, 3><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
    case 7: quantize_kernel<4, 3><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
    case 8: quantize_kernel<3, 4><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
    default: quantize_kernel<4, 4><<<unsigned(blocks), 256, 0, stream>>>(w, N, G, cb, c, s, dev_status); break;
  }
  return cudaGetLastError();
}

}  // namespace lutq
