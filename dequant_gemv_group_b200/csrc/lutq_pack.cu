// Offline restructuring of the codes and scales into layout V2 (the FLUTE
// abstract, "Daily Papers" listing: repack the quantized matrix offline so
// that the product kernel needs few bit operations to unpack, including 3-bit
// widths).
//
// One thread writes one 16-byte output word; threads are numbered in output
// order, so a warp writes 512 contiguous bytes.  The U * 32 * words_per_row
// code words come first: word id -> (tile, w, r) with r = id % 32,
// w = (id / 32) % words_per_row, tile = id / (32 * words_per_row) =
// strip * G + g.  Then the scale block of each tile, SB / 16 words: with one
// scale per group of 128 (SB = 64), word j holds slots 8 j .. 8 j + 7, slot
// 4 rq + i being row rq + 8 i; with one scale per group of 64 (SB = 128,
// scales [N, K/64]), words 0-3 hold the first 64-group's slots in that order
// and words 4-7 the second's.  Codes >= 2^bits are reported and masked.
#include "lutq_common.cuh"

namespace lutq {

__device__ __forceinline__ void load_codes(const uint8_t* p, uint8_t* out, int n) {
  // n is a multiple of 16 and p is 16-byte aligned
  for (int i = 0; i < n; i += 16) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 16; ++j) out[i + j] = uint8_t(w[j >> 2] >> (8 * (j & 3)));
  }
}

template <int BITS, int SB>
__global__ void __launch_bounds__(256)
pack_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales, int64_t N,
            int64_t K, uint4* __restrict__ packed, int32_t* dev_status) {
  constexpr int WPR = words_per_row(BITS);
  constexpr int CW = WPR * kStrip;               // code words of a tile
  constexpr int SW = SB / 16;                    // scale words of a tile
  constexpr int H = SB / kScaleBytes;            // scales per row and group of 128
  constexpr uint32_t kMask = (1u << BITS) - 1u;
  const int64_t G = K / kGroup;
  const int64_t U = (N / kStrip) * G;
  const int64_t words = U * (CW + SW);
  bool bad = false;
  for (int64_t id = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; id < words;
       id += int64_t(gridDim.x) * blockDim.x) {
    if (id >= U * CW) {
      // scale word j: slots 8 (j % 4) .. 8 (j % 4) + 7 of scale half j / 4
      const int64_t tile = (id - U * CW) / SW;
      const int j = int((id - U * CW) % SW);
      const int slot0 = 8 * (j & 3), half = j >> 2;
      const int64_t strip = tile / G, g = tile % G;
      uint32_t h[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int slot = slot0 + t, r = (slot >> 2) + 8 * (slot & 3);
        h[t] = scales[(strip * kStrip + r) * (G * H) + g * H + half];
      }
      packed[id] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                              h[6] | (h[7] << 16));
      continue;
    }
    const int r = int(id % kStrip);
    const int w = int((id / kStrip) % WPR);
    const int64_t tile = id / CW;
    const int64_t strip = tile / G, g = tile % G;
    const uint8_t* row = codes + (strip * kStrip + r) * K + g * kGroup;
    uint8_t out[16];
    if (BITS == 4) {
      uint8_t q[32];
      load_codes(row + 32 * w, q, 32);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        bad |= q[i] > kMask;
        q[i] &= kMask;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) out[i] = uint8_t(q[2 * i] | (q[2 * i + 1] << 4));
    } else if (w < 2) {
      // lo plane: 64 codes, 32 pairs; byte 4j+b = lo2(pair 8j+b) | lo2(pair 8j+4+b) << 4
      uint8_t q[64];
      load_codes(row + 64 * w, q, 64);
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        bad |= q[i] > kMask;
        q[i] &= kMask;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int p0 = 8 * j + b, p1 = 8 * j + 4 + b;
          const uint32_t lo0 = (q[2 * p0] & 3u) | ((q[2 * p0 + 1] & 3u) << 2);
          const uint32_t lo1 = (q[2 * p1] & 3u) | ((q[2 * p1 + 1] & 3u) << 2);
          out[4 * j + b] = uint8_t(lo0 | (lo1 << 4));
        }
      }
    } else {
      // hi plane over both lo words: byte 4j+b =
      //   hi2(w0, 8j+4+b) | hi2(w1, 8j+4+b) << 2 | hi2(w0, 8j+b) << 4 | hi2(w1, 8j+b) << 6
      uint8_t q[128];
      load_codes(row, q, 128);
#pragma unroll
      for (int i = 0; i < 128; ++i) q[i] &= kMask;  // range is checked by the lo-plane threads
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          uint32_t v = 0;
          const int pairs[4] = {8 * j + 4 + b, 8 * j + 4 + b, 8 * j + b, 8 * j + b};
#pragma unroll
          for (int f = 0; f < 4; ++f) {
            const int base = 64 * (f & 1) + 2 * pairs[f];
            const uint32_t h2 = (q[base] >> 2) | ((q[base + 1] >> 2) << 1);
            v |= h2 << (2 * f);
          }
          out[4 * j + b] = uint8_t(v);
        }
      }
    }
    uint4 o;
    o.x = out[0] | (out[1] << 8) | (out[2] << 16) | (uint32_t(out[3]) << 24);
    o.y = out[4] | (out[5] << 8) | (out[6] << 16) | (uint32_t(out[7]) << 24);
    o.z = out[8] | (out[9] << 8) | (out[10] << 16) | (uint32_t(out[11]) << 24);
    o.w = out[12] | (out[13] << 8) | (out[14] << 16) | (uint32_t(out[15]) << 24);
    packed[id] = o;
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) report(dev_status, LUTQ_ERR_CODE_RANGE);
}

// group64: scales [N, K/64] into 128-byte scale blocks (else [N, K/128]
// into 64-byte blocks).
cudaError_t launch_pack(const uint8_t* codes, const void* scales, int64_t N, int64_t K,
                        int bits, void* packed, int32_t* dev_status, int num_sms,
                        cudaStream_t stream, bool group64) {
  const int sb = group64 ? 2 * kScaleBytes : kScaleBytes;
  const int64_t words = (N / kStrip) * (K / kGroup) * ((tile_bytes(bits) + sb) / 16);
  int64_t blocks = (words + 255) / 256;
  const int64_t cap = int64_t(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  const uint16_t* sc = static_cast<const uint16_t*>(scales);
  uint4* out = static_cast<uint4*>(packed);
  switch ((bits == 4 ? 1 : 0) + (group64 ? 2 : 0)) {
    case 0: pack_kernel<3, 64><<<unsigned(blocks), 256, 0, stream>>>(codes, sc, N, K, out, dev_status); break;
    case 1: pack_kernel<4, 64><<<unsigned(blocks), 256, 0, stream>>>(codes, sc, N, K, out, dev_status); break;
    case 2: pack_kernel<3, 128><<<unsigned(blocks), 256, 0, stream>>>(codes, sc, N, K, out, dev_status); break;
    default: pack_kernel<4, 128><<<unsigned(blocks), 256, 0, stream>>>(codes, sc, N, K, out, dev_status); break;
  }
  return cudaGetLastError();
}

// The type blocks of a matrix with per-group data types (BitMoD abstract,
// same listing): after the U scale blocks, 8 bytes per unit t = s * G + g;
// byte rq holds the types of rows rq + 8 i (i = 0..3) of strip s, group g, in
// bits 2i+1:2i.  One thread per byte.  A type >= max_types is reported
// (LUTQ_ERR_CODE_RANGE) and stored modulo 4.
__global__ void __launch_bounds__(256)
pack_types_kernel(const uint8_t* __restrict__ types, int64_t G, int64_t bytes, int max_types,
                  uint8_t* __restrict__ out, int32_t* dev_status) {
  bool bad = false;
  for (int64_t id = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; id < bytes;
       id += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = id >> 3, rq = id & 7;
    const int64_t s = t / G, g = t % G;
    uint32_t v = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t ty = types[(s * kStrip + rq + 8 * i) * G + g];
      bad |= ty >= uint32_t(max_types);
      v |= (ty & 3u) << (2 * i);
    }
    out[id] = uint8_t(v);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) report(dev_status, LUTQ_ERR_CODE_RANGE);
}

cudaError_t launch_pack_types(const uint8_t* types, int64_t N, int64_t K, int bits, void* packed,
                              int32_t* dev_status, int num_sms, cudaStream_t stream) {
  const int64_t U = (N / kStrip) * (K / kGroup);
  const int64_t bytes = U * kTypeBytes;
  int64_t blocks = (bytes + 255) / 256;
  const int64_t cap = int64_t(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  uint8_t* out = static_cast<uint8_t*>(packed) + U * (tile_bytes(bits) + kScaleBytes);
  pack_types_kernel<<<unsigned(blocks), 256, 0, stream>>>(types, K / kGroup, bytes,
                                                          max_types(bits), out, dev_status);
  return cudaGetLastError();
}

}  // namespace lutq
