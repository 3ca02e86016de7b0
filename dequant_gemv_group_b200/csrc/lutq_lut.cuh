// The lane-duplicated pair lookup table shared by the GEMV and GEMM kernels.
//
// Shared-memory row e (256 bytes) holds, for the 8-bit pair index e, the code
// pair (c[even], c[odd]) as bf16x2: 32 copies for the "E" table at bytes
// 0..127 and 32 copies for the "O" table at bytes 128..255 (only 3-bit codes
// use O).  Lane t reads copy t, so a warp-wide lookup never has a bank
// conflict.  One byte permute forms the address (byte << 8) | lane offset.
// This is the vectorized (two codes per lookup) and duplicated table of the
// FLUTE abstract ("Daily Papers" listing, query "group-128").
#pragma once

#include <cstdint>

#include "lutq_common.cuh"

namespace lutq {

constexpr int kLutBytes = 256 * 256;  // 64 KB

// Pair (c[even], c[odd]) for index e of table `half` (0 = E, 1 = O).
//  4 bit: e = q_even | q_odd << 4.
//  3 bit, E: bits 3:0 = lo2(even) | lo2(odd) << 2, bit 4 = hi1(even), bit 5 = hi1(odd).
//  3 bit, O: bits 7:4 = lo2(even) | lo2(odd) << 2, bit 0 = hi1(even), bit 1 = hi1(odd).
template <int BITS>
__device__ __forceinline__ uint32_t lut_entry(const uint16_t* cb, int e, int half) {
  uint32_t qe, qo;
  if (BITS == 4) {
    qe = e & 15;
    qo = e >> 4;
  } else if (half == 0) {
    qe = (e & 3) | (((e >> 4) & 1) << 2);
    qo = ((e >> 2) & 3) | (((e >> 5) & 1) << 2);
  } else {
    qe = ((e >> 4) & 3) | ((e & 1) << 2);
    qo = ((e >> 6) & 3) | (((e >> 1) & 1) << 2);
  }
  return uint32_t(cb[qe]) | (uint32_t(cb[qo]) << 16);
}

// Fill the lane-duplicated table from codebooks held in registers: lane l of
// every warp passes cbw = bytes 4l .. 4l+3 of the flattened codebook array
// [types][2^BITS] (bf16 levels 2l and 2l+1, one warp-wide load for all
// tables), and each pair value is assembled with two shuffles, so no shared
// staging or barrier comes before the build (callers synchronize after it).
// Thread i builds the value of half-row i (4-bit: row i; 3-bit: row i / 2,
// half i % 2), then i + blockDim.x, ..., and stores it to the half-row's
// eight 16-byte chunks, starting at chunk i mod 8 so that each eight
// consecutive lanes cover all 32 banks.  blockDim.x is a multiple of 32, so
// all lanes of a warp take the same number of turns, as the shuffles
// require.
//
// w4_half (4-bit only): which half of each row the table goes to (0 = E, 1 =
// O); a second 4-bit table can live in the half that 4-bit codes leave free.
template <int BITS>
__device__ __forceinline__ uint32_t level_of(uint32_t cbw, int t, uint32_t q) {
  const uint32_t w = __shfl_sync(0xffffffffu, cbw, int((uint32_t(t) << (BITS - 1)) + (q >> 1)));
  return (q & 1) ? (w >> 16) : (w & 0xffffu);
}

template <int BITS>
__device__ __forceinline__ void lut_half_row(uint8_t* lut, uint32_t cbw, int t, int i,
                                             int w4_half) {
  constexpr int HALVES = BITS == 4 ? 1 : 2;
  const int e = i / HALVES, h = i % HALVES;
  uint32_t qe, qo;
  if (BITS == 4) {
    qe = e & 15;
    qo = e >> 4;
  } else if (h == 0) {
    qe = (e & 3) | (((e >> 4) & 1) << 2);
    qo = ((e >> 2) & 3) | (((e >> 5) & 1) << 2);
  } else {
    qe = ((e >> 4) & 3) | ((e & 1) << 2);
    qo = ((e >> 6) & 3) | (((e >> 1) & 1) << 2);
  }
  const uint32_t v = level_of<BITS>(cbw, t, qe) | (level_of<BITS>(cbw, t, qo) << 16);
  const uint4 v4 = make_uint4(v, v, v, v);
  uint4* half_row = reinterpret_cast<uint4*>(lut) + e * 16 + (h + w4_half) * 8;
#pragma unroll
  for (int j = 0; j < 8; ++j) half_row[(j + i) & 7] = v4;
}

template <int BITS>
__device__ __forceinline__ void build_lut_shfl(uint8_t* lut, uint32_t cbw) {
  constexpr int VALUES = 256 * (BITS == 4 ? 1 : 2);
  static_assert(VALUES % 32 == 0, "whole warps");
  for (int i = threadIdx.x; i < VALUES; i += blockDim.x) lut_half_row<BITS>(lut, cbw, 0, i, 0);
}

// The tables of per-group data types, all threads sharing the work: table t
// of 4-bit codes in row half t & 1 of the 64 KB at (t >> 1) << 16, table t of
// 3-bit codes in the 64 KB at t << 16.  A warp's lanes always work on the
// same table (its value count is a multiple of 32).
template <int BITS>
__device__ __forceinline__ void build_luts_typed(uint8_t* lut, uint32_t cbw, int types) {
  constexpr int VALUES = 256 * (BITS == 4 ? 1 : 2);
  for (int i = threadIdx.x; i < types * VALUES; i += blockDim.x) {
    const int t = i / VALUES;
    lut_half_row<BITS>(lut + ((BITS == 4 ? t >> 1 : t) << 16), cbw, t, i % VALUES,
                       BITS == 4 ? (t & 1) : 0);
  }
}

// (byte 1 of lane_off) << 16 | (byte `byte` of word) << 8 | (byte 0 of
// lane_off), with lane_off < 65536: byte 1 of lane_off selects a 64 KB table
// (per-group data types), and is zero otherwise.
__device__ __forceinline__ uint32_t lut_addr(uint32_t word, uint32_t lane_off, int byte) {
  return __byte_perm(word, lane_off, 0x6504u | (uint32_t(byte) << 4));
}

__device__ __forceinline__ uint32_t lds32(uint32_t smem_addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(smem_addr));
  return v;
}

// Four pair indices (the bytes of idx) -> four bf16x2 code pairs.  Checked
// builds compare each table offset with lut_limit (the table region's size)
// and report through st; other builds ignore both.
__device__ __forceinline__ void lookup4(uint32_t* lv, uint32_t idx, uint32_t lut_base,
                                        uint32_t lane_off, uint32_t lut_limit = 0x20000u,
                                        int32_t* st = nullptr) {
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t t = lut_addr(idx, lane_off, b);
    lv[b] = LUTQ_IN_BOUNDS(t + 4u <= lut_limit, st) ? lds32(lut_base + t) : 0u;
  }
}

// The four 32-bit index words of one 3-bit group row, j-th u32 of the two lo
// planes and of the hi plane: E/O indices of lo word 0 and lo word 1.
struct W3Index {
  uint32_t e0, o0, e1, o1;
};
__device__ __forceinline__ W3Index w3_indices(uint32_t l0, uint32_t l1, uint32_t h) {
  const uint32_t h2 = h >> 2;
  W3Index r;
  r.e0 = (l0 & 0x0F0F0F0Fu) | (h & 0xF0F0F0F0u);
  r.o0 = (l0 & 0xF0F0F0F0u) | (h & 0x0F0F0F0Fu);
  r.e1 = (l1 & 0x0F0F0F0Fu) | (h2 & 0xF0F0F0F0u);
  r.o1 = (l1 & 0xF0F0F0F0u) | (h2 & 0x0F0F0F0Fu);
  return r;
}

// Decode one row of one group (its packed words wd[0..WPR-1]) into the 64
// bf16x2 pairs of k = 0..127 in order: out[p] = (c[q[2p]], c[q[2p+1]]).
template <int BITS>
__device__ __forceinline__ void decode_group_row(uint32_t (&out)[64], const uint4 (&wd)[4],
                                                 uint32_t lut_base, uint32_t off_e,
                                                 uint32_t off_o) {
  if (BITS == 4) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t v[4] = {wd[w].x, wd[w].y, wd[w].z, wd[w].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) lookup4(out + 16 * w + 4 * j, v[j], lut_base, off_e);
    }
  } else {
    const uint32_t L0[4] = {wd[0].x, wd[0].y, wd[0].z, wd[0].w};
    const uint32_t L1[4] = {wd[1].x, wd[1].y, wd[1].z, wd[1].w};
    const uint32_t H[4] = {wd[2].x, wd[2].y, wd[2].z, wd[2].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const W3Index ix = w3_indices(L0[j], L1[j], H[j]);
      lookup4(out + 8 * j, ix.e0, lut_base, off_e);
      lookup4(out + 8 * j + 4, ix.o0, lut_base, off_o);
      lookup4(out + 32 + 8 * j, ix.e1, lut_base, off_e);
      lookup4(out + 32 + 8 * j + 4, ix.o1, lut_base, off_o);
    }
  }
}

// Half of a group row: pairs 32 h .. 32 h + 31 (k = 64 h .. 64 h + 63) into
// out[0..31].  4-bit: wd[0], wd[1] are words 2h, 2h+1.  3-bit: wd[0] is lo word
// h and wd[1] the hi word.
template <int BITS>
__device__ __forceinline__ void decode_group_half(uint32_t (&out)[32], const uint4 (&wd)[2],
                                                  int h, uint32_t lut_base, uint32_t off_e,
                                                  uint32_t off_o, uint32_t lut_limit = 0x20000u,
                                                  int32_t* st = nullptr) {
  if (BITS == 4) {
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const uint32_t v[4] = {wd[w].x, wd[w].y, wd[w].z, wd[w].w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        lookup4(out + 16 * w + 4 * j, v[j], lut_base, off_e, lut_limit, st);
    }
  } else {
    const uint32_t L[4] = {wd[0].x, wd[0].y, wd[0].z, wd[0].w};
    const uint32_t sh = 2u * uint32_t(h);
    const uint32_t H[4] = {wd[1].x >> sh, wd[1].y >> sh, wd[1].z >> sh, wd[1].w >> sh};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      lookup4(out + 8 * j, (L[j] & 0x0F0F0F0Fu) | (H[j] & 0xF0F0F0F0u), lut_base, off_e,
              lut_limit, st);
      lookup4(out + 8 * j + 4, (L[j] & 0xF0F0F0F0u) | (H[j] & 0x0F0F0F0Fu), lut_base, off_o,
              lut_limit, st);
    }
  }
}

}  // namespace lutq
