// Randomized Hadamard rotation of one 128-long group by one warp
// ("TurboQuant: A first-principles walkthrough": a randomized Hadamard
// transform can stand in for a uniform random rotation before quantizing).
//
// The group is v' = H diag(s) v with H the Sylvester Hadamard matrix of
// order 128 (H[i][j] = (-1)^popcount(i & j)).  Lane l holds v[4l .. 4l+3];
// the butterflies (a, b) -> (a + b, a - b) over the seven index bits give H
// in that order: bits 0 and 1 inside a lane, bits 2..6 across lanes
// (partner lane l ^ (1 << (bit - 2))).  T = double for the weights (their
// rotation decides the codes): the sums of bf16 inputs whose exponents span
// fewer than 38 binades are then exact and the one rounding to bf16 is that
// of the exact value.  T = float for the activations (an input of the fp32
// product): the same butterflies in fp32, a few times cheaper.
#pragma once

#include <cstdint>

namespace lutq {

template <typename T>
__device__ __forceinline__ void rht128_warp(T (&v)[4], uint32_t signs4) {
  const int lane = threadIdx.x & 31;
  // signs: byte i of signs4 is s[4 lane + i] (int8, +1 or -1)
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (int8_t(signs4 >> (8 * i)) < 0) v[i] = -v[i];
  // bit 0, then bit 1, inside the lane
  const T a = v[0] + v[1], b = v[0] - v[1], c = v[2] + v[3], d = v[2] - v[3];
  v[0] = a + c;
  v[1] = b + d;
  v[2] = a - c;
  v[3] = b - d;
  // bits 2..6 across lanes: the lane with the bit clear keeps the sum
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const T o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? o - v[i] : v[i] + o;
    }
  }
}

// The same rotation with 8 lanes per group (four groups per warp): lane l
// holds v[16 (l % 8) .. 16 (l % 8) + 15] of group l / 8, so index bits 0..3
// are inside the lane and bits 4..6 across lanes l ^ 1, l ^ 2, l ^ 4.  Every
// butterfly is the same operation on the same values, in the same bit order,
// as in rht128_warp, so the two give the same results; this one needs about
// half the instructions.  signs16: the lane's 16 signs (int8).
__device__ __forceinline__ void rht128_octet(float (&v)[16], const uint4 signs16) {
  const int lane = threadIdx.x & 31;
  const uint32_t sw[4] = {signs16.x, signs16.y, signs16.z, signs16.w};
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (int8_t(sw[i >> 2] >> (8 * (i & 3))) < 0) v[i] = -v[i];
#pragma unroll
  for (int b = 1; b < 16; b <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i & b) continue;
      const float lo = v[i], hi = v[i | b];
      v[i] = lo + hi;
      v[i | b] = lo - hi;
    }
  }
#pragma unroll
  for (int m = 1; m < 8; m <<= 1) {
    const float sgn = (lane & m) ? -1.0f : 1.0f;  // the upper lane keeps lower - upper
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = fmaf(sgn, v[i], o);
    }
  }
}

}  // namespace lutq
