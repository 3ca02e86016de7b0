// Fused dequantize-and-multiply GEMV on the CUDA cores for batches M = 1..4
// (lutq_gemv takes M = 1..16; larger batches go to the tensor-core kernel of
// lutq_gemm.cu) (the FLUTE abstract, "Daily Papers" listing, query "group-128": fuse
// dequantization with the product; duplicate and vectorize the lookup table
// against shared-memory bandwidth limits.  The BitMoD abstract, same listing:
// rescale each group's partial sum once).
//
// Work split.  The packed matrix is a sequence of
// U = (N/32) * G units, one unit = (strip of 32 rows, group of 128 codes) =
// 2048 (4-bit) or 1536 (3-bit) contiguous bytes.  A plan (choose_plan) gives
// each CTA of a grid of at most one CTA per SM a run of units: whole strips,
// an equal share of the unit sequence, or (for few, deep strips) the first or
// the last groups of strips; warp w of its NW warps takes an equal share of
// that run, so every warp streams the same number of bytes.  Sums are reduced
// in deterministic steps:
//  - a strip held whole by one warp is written by that warp;
//  - otherwise each warp leaves its partial row sums of the strips at the two
//    ends of its run in shared memory, and after a block barrier one warp per
//    strip adds them in warp order;
//  - a strip that the plan splits between two CTAs (never more) is finished
//    by whichever of the two arrives second, through one 64-bit atomic
//    exchange per row (exchange_half); a sum of two commutes, so the result
//    does not depend on which.
// Results therefore do not depend on timing.
//
// Small-batch kernel (M = 1..4).  Lane t of a warp owns the k-chunk
// q = t >> 3 (32 codes, k = 128 g + 32 q ..) of the four rows (t & 7) + 8 i,
// i = 0..3, of the strip (the 8 lanes of a quarter-warp share q, so
// activation reads are broadcasts).  Each code pair costs one byte permute
// (forming the table address) and one conflict-free shared load, shared by
// the M batch rows, then two fused multiply-adds per batch row with bf16
// multiplicands and an fp32 accumulator (a bf16 x bf16 product is exact in
// fp32, so this is the fp32 product of the widened values).  The four lanes
// of a row add their sums at the end of the strip.  Larger batches go to the
// tensor-core kernel (launch_gemv).
//
// Pipeline.  The kernel is a programmatic dependent of the work before it on
// the stream.  Its blocks start as multiprocessors free up and, before
// waiting for that work, compute their split and (the weights are read-only)
// bring weights into L2: when the plan leaves multiprocessors free, the grid
// begins with that many prefetching blocks, which land on them while the
// preceding kernel still runs and prefetch the whole matrix line by line;
// otherwise each warp prefetches its first tiles.  After the wait each block
// loads the activations into shared memory and builds the lookup table,
// and each warp keeps NB tiles (codes and scales) in flight in registers,
// loaded under one predicate so that the loop has no branch per load.
#include <cuda_bf16.h>

#include <algorithm>

#include "lutq_common.cuh"
#include "lutq_lut.cuh"
#include "lutq_rht.cuh"
#include "lutq_sm100.cuh"

namespace lutq {

constexpr int kMaxCtas = 512;           // bounds the workspace
#ifndef LUTQ_M1_WARPS
#define LUTQ_M1_WARPS 16
#endif
constexpr int kM1Warps = LUTQ_M1_WARPS; // warps per CTA of the small-batch kernel
constexpr int kMaxSmemPerBlock = 227 * 1024;

struct GemvArgs {
  const uint16_t* x;        // bf16 [M, K]
  const uint8_t* packed;    // layout V2 (codes and scales)
  const uint16_t* codebook; // bf16 [2^bits]
  float* y;                 // fp32 [M, N]
  unsigned long long* xch;  // [M][N] exchange slots of strips split between two CTAs (zero between calls)
  int32_t* status;          // caller's device status word or null
  const int8_t* signs;      // randomized Hadamard rotation of x first (null: none)
  int y_bf16;               // y is bf16 (the fp32 sums rounded once) instead of fp32
  int types;                // per-group data types: codebook holds `types` tables
                            // and the packed matrix its type blocks (0: untyped)
  int64_t N, K, G, U;       // U = number of units
  int C;                    // CTAs
  // work plan (choose_plan): kind 0 = ranges of the unit sequence, strip-
  // aligned if `align`; kind 1 = the first Cm CTAs take groups [0, G - T) of
  // one strip each, the others groups [G - T, G) of nh strips each
  uint32_t kind, align, Cm, T, nh;
  // The grid's first pf_ctas CTAs only bring the packed matrix into L2
  // (the work goes to CTAs pf_ctas .. pf_ctas + C - 1)
  uint32_t pf_ctas;
  uint32_t smem_bytes;      // the block's dynamic shared memory (checked builds)
};

// Output value i (< M N) into y; checked builds skip an index outside y.
__device__ __forceinline__ void put_y(const GemvArgs& a, int64_t i, int M, float v) {
  if (LUTQ_IN_BOUNDS(i >= 0 && i < int64_t(M) * a.N, a.status)) store_y(a.y, a.y_bf16, i, v);
}

// Part i of `parts` equal shares of [0, total): [range_begin(i), range_begin(i+1)).
// The host guarantees total * parts < 2^32, so 32-bit unsigned arithmetic is
// exact (integer division is a long instruction sequence; 64-bit even more so).
__host__ __device__ inline uint32_t range_begin(uint32_t i, uint32_t total, uint32_t parts) {
  return (i * total) / parts;
}

// The units of one CTA, in the order it takes them: strips s0, s0 + 1, ...,
// each contributing its W groups ga .. ga + W - 1; the CTA takes positions
// [v0, v1) of that sequence, position v being unit (s0 + v / W, ga + v % W).
// Every plan leaves a strip either whole in one CTA (only when W = G) or
// split between exactly two CTAs.
struct Span {
  uint32_t s0, ga, W, v0, v1;
};

__device__ __forceinline__ Span cta_span(const GemvArgs& a, uint32_t c) {
  Span p;
  const uint32_t G = uint32_t(a.G), S = uint32_t(a.N / kStrip), C = uint32_t(a.C);
  if (a.kind == 0) {
    p.s0 = 0;
    p.ga = 0;
    p.W = G;
    if (a.align) {
      p.v0 = G * range_begin(c, S, C);
      p.v1 = G * range_begin(c + 1, S, C);
    } else {
      p.v0 = range_begin(c, uint32_t(a.U), C);
      p.v1 = range_begin(c + 1, uint32_t(a.U), C);
    }
  } else if (c < a.Cm) {
    p.s0 = c;
    p.ga = 0;
    p.W = G - a.T;
    p.v0 = 0;
    p.v1 = p.W;
  } else {
    p.s0 = (c - a.Cm) * a.nh;
    p.ga = G - a.T;
    p.W = a.T;
    p.v0 = 0;
    p.v1 = p.s0 < S ? (S - p.s0 < a.nh ? S - p.s0 : a.nh) * a.T : 0u;
  }
  return p;
}

// Per-CTA table of its warps' position ranges, filled once in the prologue:
// warp w holds positions [v0 + wb[w], v0 + wb[w+1]); its first strip is ws[w].
template <int NW>
struct WarpTable {
  uint32_t wb[NW + 1];
  uint32_t ws[NW];
};

template <int NW>
__device__ __forceinline__ void fill_warp_table(WarpTable<NW>& t, const Span& p) {
  const int i = threadIdx.x;
  const uint32_t L = p.v1 - p.v0;
  if (i <= NW) t.wb[i] = range_begin(i, L, NW);
  if (i < NW) t.ws[i] = p.s0 + (p.v0 + range_begin(i, L, NW)) / p.W;
}

__device__ __forceinline__ uint32_t sm_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// A warp has summed its units of strip `strip`.  vals[i][m] is the sum of
// row rows[i] (within the strip) for batch row m, held by the lanes marked
// `writer`.  [w0, w1) are the warp's positions, first_strip the strip of w0;
// slots is its [2][M][32] shared area.  A strip held whole by the warp (which
// needs W = G) is written out; otherwise the sums wait in the slots.
template <int M, int R>
__device__ __forceinline__ void deposit_strip(const GemvArgs& a, const Span& p, uint32_t strip,
                                              uint32_t w0, uint32_t w1, uint32_t first_strip,
                                              const float (&vals)[R][M], const int (&rows)[R],
                                              bool writer, float* slots) {
  if (!writer) return;
  const uint32_t lo = (strip - p.s0) * p.W;
  if (p.W == uint32_t(a.G) && lo >= w0 && lo + p.W <= w1) {
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int m = 0; m < M; ++m)
        put_y(a, m * a.N + int64_t(strip) * kStrip + rows[i], M, vals[i][m]);
    return;
  }
  const int sl = (strip == first_strip) ? 0 : 1;
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int m = 0; m < M; ++m) slots[(sl * M + m) * kStrip + rows[i]] = vals[i][m];
}

// One of the two halves of a split row value meets the other: the first to
// arrive leaves its value (tagged in the high word) in the slot; the second
// takes it, writes the sum and clears the slot for the next call.  Both
// orders give the same fp32 sum (addition of two values commutes), so the
// result does not depend on timing.
template <int M>
__device__ __forceinline__ void exchange_half(unsigned long long* slot, float v,
                                              const GemvArgs& a, int64_t yi) {
  // one slot per output value of up to 4 batch rows (the workspace's zero part)
  if (!LUTQ_IN_BOUNDS(yi >= 0 && yi < int64_t(M) * a.N && M <= 4, a.status)) return;
  const unsigned long long mine = (1ull << 32) | __float_as_uint(v);
  const unsigned long long other = atomicExch(slot, mine);
  if (other != 0ull) {
    store_y(a.y, a.y_bf16, yi, v + __uint_as_float(uint32_t(other)));
    *slot = 0ull;
  }
}

// After a block barrier: finish every strip of the CTA's span that no single
// warp wrote out.  all_slots is [NW][2][M][32].  One warp per strip adds the
// warps' sums in warp order; a strip whole in this CTA is written, a strip
// split with the other CTA goes through exchange_half.
template <int M, int NW>
__device__ void cta_finish(const GemvArgs& a, const Span& p, const float* all_slots,
                           const WarpTable<NW>& t) {
  if (p.v0 >= p.v1) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool full = p.W == uint32_t(a.G);
  const uint32_t s_first = t.ws[0];
  const uint32_t s_last = p.s0 + (p.v1 - 1) / p.W;
  for (uint32_t strip = s_first + warp; strip <= s_last; strip += NW) {
    const uint32_t lo = (strip - p.s0) * p.W, hi = lo + p.W;
    float sum[M];
#pragma unroll
    for (int m = 0; m < M; ++m) sum[m] = 0.0f;
    // Unrolled over the warps, so that the slot reads do not wait on one
    // another; the sum still runs in warp order.  A strip held whole by one
    // warp has no other contributor (the warps' ranges are disjoint).
    bool whole = false;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const uint32_t b = p.v0 + t.wb[w], e = p.v0 + t.wb[w + 1];
      const bool some = b < e && e > lo && b < hi;   // has units of this strip
      whole |= some && b <= lo && e >= hi;           // ... all of them
      const int sl = (strip == t.ws[w]) ? 0 : 1;
      const float* src = all_slots + ((w * 2 + sl) * M) * kStrip;
#pragma unroll
      for (int m = 0; m < M; ++m) sum[m] += some ? src[m * kStrip + lane] : 0.0f;
    }
    if (full && whole) continue;  // written by its warp
    const int64_t yrow = int64_t(strip) * kStrip + lane;
    if (full && lo >= p.v0 && hi <= p.v1) {
#pragma unroll
      for (int m = 0; m < M; ++m) put_y(a, yrow + m * a.N, M, sum[m]);
      continue;
    }
    unsigned long long* xrow = a.xch + yrow;
#pragma unroll
    for (int m = 0; m < M; ++m) exchange_half<M>(xrow + m * a.N, sum[m], a, yrow + m * a.N);
  }
}


// --------------------------------------------------------------------------
// Small-batch kernel (M = 1..4)
// --------------------------------------------------------------------------

// Shared-window layout of the small-batch kernel, in addresses of the CTA's
// shared window (the block's own static shared memory and the system's
// reserved bytes lie below kSbaseMax, where dynamic shared memory begins):
//   [kLutAt, xat)                  the lookup tables: 64 KB (256 rows of 256
//                                  bytes) or, for per-group data types that
//                                  need it, 128 KB (table_region_bytes)
//   [xat, slots_at(K, M, L))       activations, bf16 in order, batch row by
//                                  batch row: a group's four chunks of 32
//                                  values (64 bytes each) are contiguous
//   [slots_at(K, M, L), small_end) warp slots, [NW][2][M][32] fp32
// with xat = kLutAt + L, L the table bytes.  The dynamic size small_end
// therefore covers the window up to the end of the slots whatever the exact
// start (<= kSbaseMax).  A table address is formed as (table << 16 | row << 8
// | column); kLutAt goes into the load's offset.
constexpr uint32_t kSbaseMax = 4096;
constexpr uint32_t kLutAt = kSbaseMax;
constexpr uint32_t kXChunkBytes = 64;
constexpr uint32_t kXGroupBytes = 4 * kXChunkBytes;

// With per-group data types, table t of 4-bit codes sits in row half t & 1
// of the 64 KB at (t >> 1) << 16, table t of 3-bit codes (both halves) in the
// 64 KB at t << 16; the address bits 23:16 come from bits 15:8 of the lane's
// column word.
__host__ __device__ constexpr uint32_t slots_at(uint32_t K, int M, uint32_t lut_bytes) {
  return kLutAt + lut_bytes + uint32_t(M) * K * 2u;  // K * 2 is a multiple of 256
}
__host__ __device__ constexpr uint32_t small_end(uint32_t K, int M, uint32_t lut_bytes) {
  return slots_at(K, M, lut_bytes) + uint32_t(kM1Warps * 2 * M * kStrip * 4);
}

// The table entry (a bf16x2 pair of levels) at table address t.
__device__ __forceinline__ uint32_t lut_ld(uint32_t t) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(t), "n"(kLutAt));
  return v;
}

// acc += c_even * x_even + c_odd * x_odd, with lv = (c_even, c_odd) and
// xw = (x_even, x_odd) bf16x2 words (low half = even k): two fused
// multiply-adds with bf16 multiplicands and an fp32 addend, one after the
// other.  The product of two bf16 values is exact in fp32, so each step
// rounds once, exactly as an fp32 fma on the widened operands would; no
// instruction widens anything.
__device__ __forceinline__ void pair_fma(float& acc, uint32_t lv, uint32_t xw) {
  asm("{\n\t.reg .b16 c0, c1, x0, x1;\n\t"
      "mov.b32 {c0, c1}, %1;\n\tmov.b32 {x0, x1}, %2;\n\t"
      "fma.rn.f32.bf16 %0, c0, x0, %0;\n\tfma.rn.f32.bf16 %0, c1, x1, %0;\n\t}"
      : "+f"(acc) : "r"(lv), "r"(xw));
}

// The same starting from zero (the first pair of a chain).
__device__ __forceinline__ void pair_first(float& acc, uint32_t lv, uint32_t xw) {
  asm("{\n\t.reg .b16 c0, c1, x0, x1;\n\t"
      "mov.b32 {c0, c1}, %1;\n\tmov.b32 {x0, x1}, %2;\n\t"
      "fma.rn.f32.bf16 %0, c0, x0, 0f00000000;\n\tfma.rn.f32.bf16 %0, c1, x1, %0;\n\t}"
      : "=f"(acc) : "r"(lv), "r"(xw));
}

// Row sums of one unit, su[i][m] for row i and batch row m.  The four rows'
// u32 index words idx[i] (four pair indices each) go against the activation
// words xq[m][0..3] of each batch row; the rows are interleaved so that four
// independent table loads and accumulator chains are in flight, and each
// table load serves all M batch rows.  FIRST starts the chains (su is not
// read).
// Checked builds compare every table address with the table region's size
// (lut_limit) and every activation address with the end of the activations
// (x_end), reporting through st; other builds ignore the three.
struct Checks {
  uint32_t lut_limit, x_end;
  int32_t* st;
};

template <bool FIRST, int M>
__device__ __forceinline__ void quad4(float (&su)[4][M], const uint32_t (&idx)[4],
                                      const uint32_t (&lc)[4], const uint32_t (&xq)[M][4],
                                      const Checks& ck) {
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    uint32_t lv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // row = byte b of the index word (bits 15:8), column = byte 0 of row
      // i's column word (bits 7:0), table = its byte 1 (bits 23:16; byte 2
      // is zero)
      const uint32_t t = __byte_perm(idx[i], lc[i], 0x6504u | (uint32_t(b) << 4));
      lv[i] = LUTQ_IN_BOUNDS(t + 4u <= ck.lut_limit, ck.st) ? lut_ld(t) : 0u;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < M; ++m) {
        if (FIRST && b == 0)
          pair_first(su[i][m], lv[i], xq[m][b]);
        else
          pair_fma(su[i][m], lv[i], xq[m][b]);
      }
  }
}

// Four activation words (8 bf16 values) of each batch row: batch row m's
// run of the current group starts at xa + m * xstride.
template <int M>
__device__ __forceinline__ void load_xq(uint32_t (&xq)[M][4], uint32_t xa, uint32_t xstride,
                                        const Checks& ck) {
#pragma unroll
  for (int m = 0; m < M; ++m) {
    if (!LUTQ_IN_BOUNDS(xa + uint32_t(m) * xstride + 16u <= ck.x_end, ck.st)) {
      xq[m][0] = xq[m][1] = xq[m][2] = xq[m][3] = 0u;
      continue;
    }
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(xq[m][0]), "=r"(xq[m][1]), "=r"(xq[m][2]), "=r"(xq[m][3])
                 : "r"(xa + uint32_t(m) * xstride));
  }
}

// Byte offset, inside a tile, of the lane's packed bytes of row rq; rows
// rq + 8 i follow at +128 i.  4-bit: word q.  3-bit: u32 pair 2 (q & 1) of lo
// word q >> 1 (its hi-plane bytes are lane_hi_delta(q) further on).
template <int BITS>
__device__ __forceinline__ uint32_t lane_tile_offset(int q, int rq) {
  return BITS == 4 ? uint32_t((32 * q + rq) * kWordBytes)
                   : uint32_t((32 * (q >> 1) + rq) * kWordBytes + 8 * (q & 1));
}
__device__ __forceinline__ uint32_t lane_hi_delta(int q) {
  return uint32_t((64 - 32 * (q >> 1)) * kWordBytes);
}

// The lane's share of one unit, loaded only if live > 0 (otherwise nothing is
// read and the registers are left as they are): row i's 16 bytes of the tile
// at p (4-bit: one word; 3-bit: 8 lo-plane bytes, then the 8 hi-plane bytes
// hi_delta further on) into wd[i], and the scales of rows 0..3 (bf16 pairs:
// rows 0, 1 and rows 2, 3) from ps into sv.  One predicate serves all loads.
template <int BITS>
__device__ __forceinline__ void fetch_unit(uint4 (&wd)[4], uint32_t (&sv)[2], const uint8_t* p,
                                           uint32_t hi_delta, const uint8_t* ps, int live) {
  if (BITS == 4) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.gt.s32 p, %20, 0;\n\t"
        "@p ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%18];\n\t"
        "@p ld.global.nc.L1::no_allocate.v4.u32 {%4, %5, %6, %7}, [%18+128];\n\t"
        "@p ld.global.nc.L1::no_allocate.v4.u32 {%8, %9, %10, %11}, [%18+256];\n\t"
        "@p ld.global.nc.L1::no_allocate.v4.u32 {%12, %13, %14, %15}, [%18+384];\n\t"
        "@p ld.global.nc.v2.u32 {%16, %17}, [%19];\n\t}"
        : "=r"(wd[0].x), "=r"(wd[0].y), "=r"(wd[0].z), "=r"(wd[0].w), "=r"(wd[1].x),
          "=r"(wd[1].y), "=r"(wd[1].z), "=r"(wd[1].w), "=r"(wd[2].x), "=r"(wd[2].y),
          "=r"(wd[2].z), "=r"(wd[2].w), "=r"(wd[3].x), "=r"(wd[3].y), "=r"(wd[3].z),
          "=r"(wd[3].w), "=r"(sv[0]), "=r"(sv[1])
        : "l"(p), "l"(ps), "r"(live));
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.gt.s32 p, %21, 0;\n\t"
        "@p ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%18];\n\t"
        "@p ld.global.nc.v2.u32 {%2, %3}, [%19];\n\t"
        "@p ld.global.nc.L1::no_allocate.v2.u32 {%4, %5}, [%18+128];\n\t"
        "@p ld.global.nc.v2.u32 {%6, %7}, [%19+128];\n\t"
        "@p ld.global.nc.L1::no_allocate.v2.u32 {%8, %9}, [%18+256];\n\t"
        "@p ld.global.nc.v2.u32 {%10, %11}, [%19+256];\n\t"
        "@p ld.global.nc.L1::no_allocate.v2.u32 {%12, %13}, [%18+384];\n\t"
        "@p ld.global.nc.v2.u32 {%14, %15}, [%19+384];\n\t"
        "@p ld.global.nc.v2.u32 {%16, %17}, [%20];\n\t}"
        : "=r"(wd[0].x), "=r"(wd[0].y), "=r"(wd[0].z), "=r"(wd[0].w), "=r"(wd[1].x),
          "=r"(wd[1].y), "=r"(wd[1].z), "=r"(wd[1].w), "=r"(wd[2].x), "=r"(wd[2].y),
          "=r"(wd[2].z), "=r"(wd[2].w), "=r"(wd[3].x), "=r"(wd[3].y), "=r"(wd[3].z),
          "=r"(wd[3].w), "=r"(sv[0]), "=r"(sv[1])
        : "l"(p), "l"(p + hi_delta), "l"(ps), "r"(live));
  }
}

// The lane's type byte of one unit (per-group data types), loaded only if
// live > 0.
__device__ __forceinline__ void fetch_type_byte(uint32_t& ty, const uint8_t* p, int live) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.gt.s32 p, %2, 0;\n\t@p ld.global.nc.u8 %0, [%1];\n\t}"
      : "+r"(ty) : "l"(p), "r"(live));
}

// Row sums of one unit for the lane's four rows and the M batch rows; xa is
// the address of the lane's 32 activations of the group for batch row 0.
template <int BITS, int M>
__device__ __forceinline__ void unit_partial(float (&su)[4][M], const uint4 (&wd)[4],
                                             const uint32_t (&lce)[4], const uint32_t (&lco)[4],
                                             uint32_t hi_shift,
                                             uint32_t xa, uint32_t xstride, const Checks& ck) {
  uint32_t xq[M][4];
  if (BITS == 4) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      load_xq<M>(xq, xa + 16u * j, xstride, ck);
      const uint32_t idx[4] = {j == 0 ? wd[0].x : j == 1 ? wd[0].y : j == 2 ? wd[0].z : wd[0].w,
                               j == 0 ? wd[1].x : j == 1 ? wd[1].y : j == 2 ? wd[1].z : wd[1].w,
                               j == 0 ? wd[2].x : j == 1 ? wd[2].y : j == 2 ? wd[2].z : wd[2].w,
                               j == 0 ? wd[3].x : j == 1 ? wd[3].y : j == 2 ? wd[3].z : wd[3].w};
      if (j == 0)
        quad4<true, M>(su, idx, lce, xq, ck);
      else
        quad4<false, M>(su, idx, lce, xq, ck);
    }
  } else {
    // lo u32 j goes with hi u32 j; lo word 1 reads its hi fields two bits up
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t e[4], o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t l = j == 0 ? wd[i].x : wd[i].y;
        const uint32_t h = (j == 0 ? wd[i].z : wd[i].w) >> hi_shift;
        e[i] = (l & 0x0F0F0F0Fu) | (h & 0xF0F0F0F0u);
        o[i] = (l & 0xF0F0F0F0u) | (h & 0x0F0F0F0Fu);
      }
      load_xq<M>(xq, xa + 32u * j, xstride, ck);
      if (j == 0)
        quad4<true, M>(su, e, lce, xq, ck);
      else
        quad4<false, M>(su, e, lce, xq, ck);
      load_xq<M>(xq, xa + 32u * j + 16u, xstride, ck);
      quad4<false, M>(su, o, lco, xq, ck);
    }
  }
}

// Prefetch depth NB: tiles in registers ahead of the one being consumed.
// Two when prefetching blocks have brought the weights into L2 (a third
// buffer measured 2% slower on the 4096 x 14336 layer); three for a single
// batch row whose weights come from HBM (4% faster on 8192 x 28672, 3 bit).

// base + i * scale as one wide multiply-add (i, scale 32-bit).
template <typename T>
__device__ __forceinline__ const T* wide_addr(const T* base, uint32_t i, uint32_t scale) {
  uint64_t r;
  asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(r) : "r"(i), "r"(scale), "l"(base));
  return reinterpret_cast<const T*>(r);
}

__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_cg_u32(const uint16_t* p) {
  uint32_t r;
  asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// TREG: 0 without per-group data types; 1 or 2 with them, the table region
// being TREG x 64 KB (table_region_bytes).  SB: bytes of a unit's scale
// block, 64 (one scale per group of 128) or 128 (one per group of 64: the
// lane's 32 codes lie in 64-group q >> 1, whose scales are the block's
// half q >> 1).
template <int BITS, int M, int NB, int TREG, int SB = kScaleBytes>
__global__ void __launch_bounds__(kM1Warps * 32, 1) gemv_small_kernel(GemvArgs a) {
  constexpr bool TYPED = TREG > 0;
  static_assert(SB == kScaleBytes || !TYPED, "per-group types use 64-byte scale blocks");
  constexpr int TB = tile_bytes(BITS);
  constexpr int UB = TB + SB + (TYPED ? kTypeBytes : 0);  // packed bytes per unit
  constexpr uint32_t kLutRegion = TREG == 2 ? 0x20000u : 0x10000u;
  constexpr uint32_t kXAt = kLutAt + kLutRegion;
  // Table-select bits a lookup may use: with one 64 KB region only the row
  // half (4-bit codes), so every address stays inside the tables whatever
  // type a group stores (a type >= types reads an unfilled table).
  constexpr uint32_t sel_mask = (BITS == 4 ? 0x080u : 0u) | (TREG == 2 ? 0x100u : 0u);
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ WarpTable<kM1Warps> wt;
  const uint32_t sbase = sm_addr(smem);
  const uint32_t G = uint32_t(a.G), K = uint32_t(a.K);
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;

  // A grid smaller than the GPU starts with pf_ctas CTAs that find free
  // multiprocessors while the preceding kernel on the stream still runs:
  // they bring the whole packed matrix into L2, line by line, and leave (a
  // prefetch reads nothing into the kernel, so it needs no wait for the
  // preceding kernel).
  if (blockIdx.x < a.pf_ctas) {
    const uint32_t lines = uint32_t((uint64_t(a.U) * UB + 127u) / 128u);
    for (uint32_t j = blockIdx.x * blockDim.x + threadIdx.x; j < lines;
         j += a.pf_ctas * blockDim.x)
      prefetch_l2(a.packed + uint64_t(j) * 128u);
    return;
  }
  const Span sp = cta_span(a, blockIdx.x - a.pf_ctas);
  // the warp's positions [u0, u1) of the CTA's unit sequence
  const uint32_t u0 = sp.v0 + range_begin(wl, sp.v1 - sp.v0, kM1Warps);
  const uint32_t u1 = sp.v0 + range_begin(wl + 1, sp.v1 - sp.v0, kM1Warps);
  const uint32_t first_strip = sp.s0 + u0 / sp.W;
  const uint32_t g_first = u0 % sp.W;  // within the window: group sp.ga + g_first
  const int q = lane >> 3, rq = lane & 7;

  // Fetch cursor, in the order of the positions: tile index ft (strip * G +
  // group) of the next unit to load; fleft units until the end of the window
  // in that strip (the window's first group of the next strip follows); fn
  // units still to load.
  uint32_t ft = first_strip * G + sp.ga + g_first;
  uint32_t fleft = sp.W - g_first;
  int fn = int(u1 - u0);
  const uint32_t lane_off = lane_tile_offset<BITS>(q, rq);
  const uint32_t hi_delta = BITS == 3 ? lane_hi_delta(q) : 0u;
  const uint8_t* const pk = a.packed + lane_off;
  // the scales of the lane's rows rq + 8 i, i = 0..3: 8 bytes of each unit's
  // 64 (of the half of the 128 that holds the lane's 64-group)
  const uint8_t* const psc =
      a.packed + uint64_t(a.U) * TB + scale_slot(rq) + (SB > kScaleBytes ? 64 * (q >> 1) : 0);
  // per-group types: byte rq of each unit's 8 (rows rq + 8 i in bits 2i+1:2i)
  const uint8_t* const pty = a.packed + uint64_t(a.U) * (TB + kScaleBytes) + rq;

  // Before the preceding kernel on the stream is complete (this kernel is
  // its programmatic dependent) nothing is read.  Without prefetching CTAs,
  // the warp's first tiles are brought into L2 (which keeps no stale copy)
  // meanwhile; the values are loaded after the wait below.
  if (a.pf_ctas == 0 && u0 < u1) {
    uint32_t t = ft, l = fleft;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      if (u0 + j < u1) {
        const uint8_t* p = wide_addr(pk, t, uint32_t(TB));
#pragma unroll
        for (int i = 0; i < 4; ++i) prefetch_l2(p + 128 * i);
        if (lane == 0 || (SB > kScaleBytes && lane == 16))
          prefetch_l2(wide_addr(psc, t, uint32_t(SB)));
        if (TYPED && lane == 0) prefetch_l2(wide_addr(pty, t, uint32_t(kTypeBytes)));
      }
      ++t;
      if (--l == 0) {
        t += G - sp.W;
        l = sp.W;
      }
    }
  }
  if (threadIdx.x == 0) prefetch_l2(a.codebook);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // The layout needs dynamic shared memory to begin below kSbaseMax; the
  // host allocates for that.  Should it not, nothing is touched.
  if (sbase > kSbaseMax) {
    if (threadIdx.x == 0) report(a.status, LUTQ_ERR_CUDA);
    return;
  }
  // checked builds: the window (tables, activations, slots) lies inside the
  // block's dynamic shared memory
  if (!LUTQ_IN_BOUNDS(small_end(K, M, kLutRegion) - sbase <= a.smem_bytes, a.status)) return;

  auto fetch = [&](uint4 (&wd)[4], uint32_t (&sv)[2], uint32_t& ty) {
    // checked builds: a unit past the packed matrix is not loaded
    int live = fn;
    if (fn > 0 && !LUTQ_IN_BOUNDS(ft < uint32_t(a.U), a.status)) live = 0;
    fetch_unit<BITS>(wd, sv, wide_addr(pk, ft, TB), hi_delta,
                     wide_addr(psc, ft, uint32_t(SB)), live);
    if (TYPED) fetch_type_byte(ty, wide_addr(pty, ft, uint32_t(kTypeBytes)), live);
    --fn;
    ++ft;
    if (--fleft == 0) {  // on to the window's first group of the next strip
      ft += G - sp.W;
      fleft = sp.W;
    }
  };

  // The activations first (all threads, 16 bytes at a time, through L2:
  // the preceding kernel may have written them), the codebook (lane t holds
  // codebook[t mod 2^BITS], and the table is built from it with shuffles)
  // and the first tile; the other NB - 1 tiles once the activations are in.
  uint4 buf[NB][4];
  uint32_t sbuf[NB][2];
  uint32_t tbuf[NB];
#pragma unroll
  for (int t = 0; t < NB; ++t) tbuf[t] = 0;
  uint32_t cbw = 0;  // bytes 4 lane .. 4 lane + 3 of the codebook array
  {
    constexpr uint32_t kStep = kM1Warps * 32 * 16;
    const uint32_t xbytes = uint32_t(M) * K * 2u;
    const uint8_t* xg = reinterpret_cast<const uint8_t*>(a.x);
    uint8_t* xs = smem + (kXAt - sbase);
    uint32_t o = threadIdx.x * 16u;
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (o + j * kStep < xbytes) v[j] = ld_cg_v4(xg + o + j * kStep);
    // all tables in one warp-wide load (at most 128 bytes)
    if (lane < ((TYPED ? a.types : 1) << (BITS - 1))) cbw = ld_cg_u32(a.codebook + 2 * lane);
    fetch(buf[0], sbuf[0], tbuf[0]);
    for (;;) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (o + j * kStep < xbytes) *reinterpret_cast<uint4*>(xs + o + j * kStep) = v[j];
      o += 4 * kStep;
      if (o >= xbytes) break;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (o + j * kStep < xbytes) v[j] = ld_cg_v4(xg + o + j * kStep);
    }
  }
  if (TYPED)
    build_luts_typed<BITS>(smem + (kLutAt - sbase), cbw, a.types);
  else
    build_lut_shfl<BITS>(smem + (kLutAt - sbase), cbw);
#pragma unroll
  for (int t = 1; t < NB; ++t) fetch(buf[t], sbuf[t], tbuf[t]);
  if (a.signs != nullptr) {
    // Rotate every 128-long group of the activations in place, eight lanes
    // per group: x_g <- H diag(s) x_g / 128, fp32 butterflies (as
    // lutq_rht_activations), rounded once to bf16 (group t = m G + g of
    // batch row m sits at 256 t).
    const uint4 signs16 = reinterpret_cast<const uint4*>(a.signs)[lane & 7];
    __syncthreads();  // the block's activation stores
    uint8_t* xs = smem + (kXAt - sbase);
    const uint32_t groups = uint32_t(M) * G;
    for (uint32_t t0 = 4u * uint32_t(wl); t0 < groups; t0 += 4u * kM1Warps) {
      const uint32_t t = t0 + uint32_t(lane >> 3);
      uint4* p = reinterpret_cast<uint4*>(xs + t * kXGroupBytes + 32u * uint32_t(lane & 7));
      uint4 r0 = make_uint4(0, 0, 0, 0), r1 = r0;
      if (t < groups) {
        r0 = p[0];
        r1 = p[1];
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
        h[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i] * (1.0f / kGroup))) |
               (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i + 1] * (1.0f / kGroup))))
                << 16);
      if (t < groups) {
        p[0] = make_uint4(h[0], h[1], h[2], h[3]);
        p[1] = make_uint4(h[4], h[5], h[6], h[7]);
      }
    }
  }
  __syncthreads();  // table, activations

  const uint32_t lane_e = uint32_t(lane) * 4u, lane_o = 128u + uint32_t(lane) * 4u;
  const uint32_t hi_shift = BITS == 3 ? 2u * uint32_t(q >> 1) : 0u;
  float* const slots = reinterpret_cast<float*>(
      smem + (slots_at(K, M, kLutRegion) - sbase));
  float* const my_slots = slots + wl * 2 * M * kStrip;
  int rows[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) rows[i] = rq + 8 * i;
  const uint32_t xstride = K * 2u;
  const Checks ck = {kLutRegion, kXAt + uint32_t(M) * xstride, a.status};
  // the lane's activations of the window's first group, batch row 0
  const uint32_t xa_w = kXAt + sp.ga * kXGroupBytes + uint32_t(q) * kXChunkBytes;

  if (u0 < u1) {
    uint32_t strip = first_strip;
    uint32_t xa = xa_w + g_first * kXGroupBytes;
    // cleft: units of the current strip still to consume; rest: units of
    // the range after the current strip's
    uint32_t cleft = min(sp.W - g_first, u1 - u0);
    uint32_t rest = (u1 - u0) - cleft;
    float acc[4][M];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < M; ++m) acc[i][m] = 0.0f;
    // Consume the unit held in (wd, sv); true once the range is done.
    auto step = [&](const uint4 (&wd)[4], const uint32_t (&sv)[2], uint32_t ty) -> bool {
      // each row's column words: the lane's column, and with per-group types
      // the row's table (4-bit: type bit 0 -> address bit 7, bit 1 -> bit 16;
      // 3-bit: type bit 0 -> bit 16)
      uint32_t lce[4], lco[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t sel = 0;
        if (TYPED)
          sel = (BITS == 4 ? (ty << 7) >> (2 * i) : (ty << 8) >> (2 * i)) & sel_mask;
        lce[i] = lane_e | sel;
        lco[i] = lane_o | sel;
      }
      if (TYPED) {
        // a group whose stored type has no table in this call is reported
        // (its lookups stay inside the allocated tables)
        const uint32_t T = uint32_t(a.types);
        if ((ty & 3u) >= T || ((ty >> 2) & 3u) >= T || ((ty >> 4) & 3u) >= T ||
            ((ty >> 6) & 3u) >= T)
          report(a.status, LUTQ_ERR_CODE_RANGE);
      }
      float su[4][M];
      unit_partial<BITS, M>(su, wd, lce, lco, hi_shift, xa, xstride, ck);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float s = (i & 1) ? bf16_hi_to_f32(sv[i >> 1]) : bf16_lo_to_f32(sv[i >> 1]);
#pragma unroll
        for (int m = 0; m < M; ++m) acc[i][m] = fmaf(s, su[i][m], acc[i][m]);
      }
      xa += kXGroupBytes;
      if (--cleft != 0) return false;
      // the warp's units of this strip are summed: the four lanes of a row
      // add theirs, and the strip's sums are written or left in the slots
      float vals[4][M];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < M; ++m) {
          float v = acc[i][m];
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          vals[i][m] = v;
          acc[i][m] = 0.0f;
        }
      deposit_strip<M, 4>(a, sp, strip, u0, u1, first_strip, vals, rows, q == 0, my_slots);
      if (rest == 0) return true;
      ++strip;
      xa = xa_w;
      cleft = min(sp.W, rest);
      rest -= cleft;
      return false;
    };
    for (;;) {
#pragma unroll
      for (int t = 0; t < NB; ++t) {
        if (step(buf[t], sbuf[t], tbuf[t])) goto range_done;
        fetch(buf[t], sbuf[t], tbuf[t]);
      }
    }
  range_done:;
  }
  fill_warp_table<kM1Warps>(wt, sp);
  __syncthreads();
  cta_finish<M, kM1Warps>(a, sp, slots, wt);
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------

// One 8-byte exchange slot per output value (exchange_half).
int64_t gemv_workspace_bytes(int64_t M, int64_t N) { return (M * N * 8 + 255) / 256 * 256; }

// Per device: the largest dynamic shared-memory size already granted to a
// kernel instance.
struct SmemGrant {
  int bytes[64] = {0};
};

template <typename Kernel>
static cudaError_t grant_smem(Kernel k, SmemGrant& g, int smem) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g.bytes[dev] < smem) {
    err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    g.bytes[dev] = smem;
  }
  return cudaSuccess;
}

// The work plan (see cta_span).  Costs are in units per CTA, the longest CTA
// deciding; a plan that splits strips between two CTAs pays kExchangeUnits
// more for the exchange of the split halves at the end and the extra strip
// ends (measured: main/helper CTAs of 98 units run as fast as whole strips
// of 112, and 16 + 15 units beat 32 whole ones).
//  - whole strips, dealt out in equal runs to min(SMs, strips) CTAs;
//  - equal unit ranges, one CTA per SM, when there are at least as many
//    strips as CTAs (each range then spans a strip or more, so a strip is
//    split between two CTAs at most);
//  - otherwise, main and helper CTAs: one CTA per strip takes its first
//    G - T groups, and each of the remaining CTAs the last T groups of nh
//    strips, T balancing the two.
constexpr int64_t kExchangeUnits = 15;

struct Plan {
  int C;
  uint32_t kind, align, Cm, T, nh;
};

static Plan choose_plan(int64_t S, int64_t G, int num_sms) {
  const int64_t cap = std::min<int64_t>(num_sms, kMaxCtas);
  const int64_t U = S * G;
  Plan best;
  // whole strips
  best.C = int(std::min<int64_t>(cap, S));
  best.kind = 0;
  best.align = 1;
  best.Cm = best.T = best.nh = 0;
  int64_t t_best = (S + best.C - 1) / best.C * G;
  if (S >= cap) {
    const int64_t t = (U + cap - 1) / cap + kExchangeUnits;
    if (t < t_best) {
      t_best = t;
      best.C = int(cap);
      best.align = 0;
    }
  } else if (G >= 2) {
    const int64_t H = cap - S;
    const int64_t nh = (S + H - 1) / H;
    int64_t T = (G + nh) / (nh + 1);  // G / (nh + 1), rounded
    T = std::max<int64_t>(1, std::min<int64_t>(T, G - 1));
    const int64_t t = std::max<int64_t>(G - T, nh * T) + kExchangeUnits;
    if (t < t_best) {
      t_best = t;
      best.C = int(S + (S + nh - 1) / nh);
      best.kind = 1;
      best.align = 0;
      best.Cm = uint32_t(S);
      best.T = uint32_t(T);
      best.nh = uint32_t(nh);
    }
  }
  return best;
}

// The plan as six integers {C, kind, align, Cm, T, nh} (for inspection).
void gemv_plan(int64_t N, int64_t K, int num_sms, int32_t* out) {
  const Plan pl = choose_plan(N / kStrip, K / kGroup, num_sms);
  out[0] = pl.C;
  out[1] = int32_t(pl.kind);
  out[2] = int32_t(pl.align);
  out[3] = int32_t(pl.Cm);
  out[4] = int32_t(pl.T);
  out[5] = int32_t(pl.nh);
}

// A packed matrix up to this size is brought into L2
// ahead of the loads by prefetching CTAs on the multiprocessors the plan
// leaves free.
constexpr int64_t kPrefetchBytes = int64_t(64) << 20;

static void apply_plan(GemvArgs& a, int num_sms, int bits, int sb) {
  const int64_t unit_bytes = tile_bytes(bits) + sb + (a.types > 0 ? kTypeBytes : 0);
  const Plan pl = choose_plan(a.N / kStrip, a.G, num_sms);
  a.C = pl.C;
  a.kind = pl.kind;
  a.align = pl.align;
  a.Cm = pl.Cm;
  a.T = pl.T;
  a.nh = pl.nh;
  const int64_t bytes = a.U * unit_bytes;
  a.pf_ctas = pl.C < num_sms && bytes <= kPrefetchBytes ? uint32_t(num_sms - pl.C) : 0u;
}


static int64_t small_smem(int64_t K, int M, int lut_bytes) {
  return K < (int64_t(1) << 20) ? int64_t(small_end(uint32_t(K), M, uint32_t(lut_bytes)))
                                : int64_t(1) << 30;
}

template <int BITS, int M, int TREG, int SB = kScaleBytes>
static cudaError_t launch_small(GemvArgs a, int num_sms, cudaStream_t stream) {
  constexpr bool TYPED = TREG > 0;
  static SmemGrant grant2, grant3;
  const int smem = int(small_smem(a.K, M, TREG == 2 ? 0x20000 : 0x10000));
  apply_plan(a, num_sms, BITS, SB);
  constexpr int kDeep = M == 1 && !TYPED ? 3 : 2;
  const bool deep = M == 1 && !TYPED && a.pf_ctas == 0;
  auto kernel = deep ? gemv_small_kernel<BITS, M, kDeep, TREG, SB>
                     : gemv_small_kernel<BITS, M, 2, TREG, SB>;
  cudaError_t err = grant_smem(kernel, deep ? grant3 : grant2, smem);
  if (err != cudaSuccess) return err;
  // programmatic dependent launch: the prefetching blocks and the work
  // blocks' set-up may overlap the end of the preceding kernel on the stream
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(a.C) + a.pf_ctas);
  cfg.blockDim = dim3(kM1Warps * 32);
  cfg.dynamicSmemBytes = size_t(smem);
  a.smem_bytes = uint32_t(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

cudaError_t launch_gemm(const void* x, int64_t M, const void* packed, const void* codebook,
                        int bits, int64_t N, int64_t K, float* y, void* workspace,
                        int32_t* dev_status, int num_sms, cudaStream_t stream, int types = 0,
                        bool y_bf16 = false, int64_t zero_bytes = -1, bool group64 = false);

// Batches up to kMaxSmallBatch run on the CUDA cores when their activations
// fit the small-batch kernel's shared memory.  Larger batches are a dense
// contraction for the CUDA cores (each table lookup feeds 2M multiply-adds;
// from M = 5 on that costs more than the tensor-core kernel's whole pass),
// so they, and over-long rows, take the tcgen05 kernel of lutq_gemm.
constexpr int kMaxSmallBatch = 4;

static bool small_fits(int64_t M, int64_t K, int lut_bytes = 0x10000) {
  return M >= 1 && M <= kMaxSmallBatch &&
         small_smem(K, int(M), lut_bytes) <= kMaxSmemPerBlock - 1024;
}

template <int BITS, int TREG = 0, int SB = kScaleBytes>
static cudaError_t launch_bits(const GemvArgs& a, int M, int num_sms, cudaStream_t s) {
  switch (M) {
    case 1: return launch_small<BITS, 1, TREG, SB>(a, num_sms, s);
    case 2: return launch_small<BITS, 2, TREG, SB>(a, num_sms, s);
    case 3: return launch_small<BITS, 3, TREG, SB>(a, num_sms, s);
    default: return launch_small<BITS, 4, TREG, SB>(a, num_sms, s);
  }
}

cudaError_t launch_gemv(const void* x, int64_t M, const void* packed, const void* codebook,
                        int bits, int64_t N, int64_t K, float* y, void* workspace,
                        int32_t* dev_status, int num_sms, cudaStream_t stream, bool y_bf16,
                        int64_t zero_bytes, bool group64) {
  GemvArgs a;
  a.y_bf16 = y_bf16 ? 1 : 0;
  a.x = static_cast<const uint16_t*>(x);
  a.packed = static_cast<const uint8_t*>(packed);
  a.codebook = static_cast<const uint16_t*>(codebook);
  a.y = y;
  a.xch = static_cast<unsigned long long*>(workspace);
  a.status = dev_status;
  a.signs = nullptr;
  a.types = 0;
  a.N = N;
  a.K = K;
  a.G = K / kGroup;
  a.U = (N / kStrip) * a.G;
  a.C = 0;
  // unit indices and range arithmetic are 32-bit (U * CTAs < 2^32)
  if (a.U * kMaxCtas >= (int64_t(1) << 32)) return cudaErrorInvalidValue;
  if (!small_fits(M, K))
    return launch_gemm(x, M, packed, codebook, bits, N, K, y, workspace, dev_status,
                       num_sms, stream, 0, y_bf16, zero_bytes, group64);
  if (group64)
    return bits == 4 ? launch_bits<4, 0, 2 * kScaleBytes>(a, int(M), num_sms, stream)
                     : launch_bits<3, 0, 2 * kScaleBytes>(a, int(M), num_sms, stream);
  return bits == 4 ? launch_bits<4>(a, int(M), num_sms, stream)
                   : launch_bits<3>(a, int(M), num_sms, stream);
}

// Whether lutq_gemv runs an M x K product on the CUDA-core kernel.
bool gemv_small_path(int64_t M, int64_t K, int bits) {
  (void)bits;
  return small_fits(M, K);
}

// Whether lutq_gemv_typed runs an M x K product on the CUDA-core kernel (with
// the table region that `types` tables need).
bool gemv_typed_path(int64_t M, int64_t K, int bits, int types) {
  return small_fits(M, K, table_region_bytes(bits, types));
}

// lutq_gemv with the activations rotated in the kernel's prologue; only for
// the CUDA-core kernel (the caller checks gemv_small_path).
cudaError_t launch_gemv_rht(const void* x, int64_t M, const void* packed, const void* codebook,
                            const int8_t* signs, int bits, int64_t N, int64_t K, float* y,
                            void* workspace, int32_t* dev_status, int num_sms,
                            cudaStream_t stream) {
  if (!gemv_small_path(M, K, bits)) return cudaErrorInvalidValue;
  GemvArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.packed = static_cast<const uint8_t*>(packed);
  a.codebook = static_cast<const uint16_t*>(codebook);
  a.y = y;
  a.xch = static_cast<unsigned long long*>(workspace);
  a.status = dev_status;
  a.signs = signs;
  a.y_bf16 = 0;
  a.types = 0;
  a.N = N;
  a.K = K;
  a.G = K / kGroup;
  a.U = (N / kStrip) * a.G;
  a.C = 0;
  if (a.U * kMaxCtas >= (int64_t(1) << 32)) return cudaErrorInvalidValue;
  return bits == 4 ? launch_bits<4>(a, int(M), num_sms, stream)
                   : launch_bits<3>(a, int(M), num_sms, stream);
}

// lutq_gemv with per-group data types: `codebooks` holds `types` tables of
// 2^bits levels and `packed` the type blocks.  The CUDA-core kernel (with its
// 128 KB table region) where it fits, the tensor-core kernel otherwise.
cudaError_t launch_gemv_typed(const void* x, int64_t M, const void* packed, const void* codebooks,
                              int types, int bits, int64_t N, int64_t K, float* y,
                              void* workspace, int32_t* dev_status, int num_sms,
                              cudaStream_t stream) {
  if (types < 1 || types > max_types(bits)) return cudaErrorInvalidValue;
  if (!gemv_typed_path(M, K, bits, types))
    return launch_gemm(x, M, packed, codebooks, bits, N, K, y, workspace, dev_status, num_sms,
                       stream, types);
  GemvArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.packed = static_cast<const uint8_t*>(packed);
  a.codebook = static_cast<const uint16_t*>(codebooks);
  a.y = y;
  a.xch = static_cast<unsigned long long*>(workspace);
  a.status = dev_status;
  a.signs = nullptr;
  a.y_bf16 = 0;
  a.types = types;
  a.N = N;
  a.K = K;
  a.G = K / kGroup;
  a.U = (N / kStrip) * a.G;
  a.C = 0;
  if (a.U * kMaxCtas >= (int64_t(1) << 32)) return cudaErrorInvalidValue;
  if (table_region_bytes(bits, types) > 0x10000)
    return bits == 4 ? launch_bits<4, 2>(a, int(M), num_sms, stream)
                     : launch_bits<3, 2>(a, int(M), num_sms, stream);
  return bits == 4 ? launch_bits<4, 1>(a, int(M), num_sms, stream)
                   : launch_bits<3, 1>(a, int(M), num_sms, stream);
}

}  // namespace lutq
