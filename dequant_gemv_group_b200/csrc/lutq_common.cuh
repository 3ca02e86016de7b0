// Shared helpers for the liblutq kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "lutq.h"

namespace lutq {

constexpr int kGroup = 128;      // weights per quantization group along K
constexpr int kStrip = 32;       // rows per packing strip (layout V2)
constexpr int kWordBytes = 16;   // one packed word = one 16-byte vector load
constexpr int kScaleBytes = 64;  // one unit's 32 row scales

// Layout V2: unit t (strip of 32 rows, group of 128 codes) has tile_bytes of
// codes at t * tile_bytes and its scales at U * tile_bytes + t * 64, row r's
// at byte scale_slot(r) of those 64.
__host__ __device__ constexpr int tile_bytes(int bits) { return bits == 4 ? 2048 : 1536; }
__host__ __device__ constexpr int scale_slot(int r) { return 2 * (4 * (r & 7) + (r >> 3)); }
__host__ __device__ constexpr int words_per_row(int bits) { return bits == 4 ? 4 : 3; }

// Per-group data types: up to 4 codebooks with 4-bit codes, 2 with 3-bit
// codes (the kernels' tables must fit shared memory); a matrix packed with
// types carries 8 type bytes per unit after the scale blocks.
constexpr int kTypeBytes = 8;
__host__ __device__ constexpr int max_types(int bits) { return bits == 4 ? 4 : 2; }

// Bytes of the lookup-table region in shared memory: one 64 KB region of 256
// rows of 256 bytes (4-bit codes use the first half of each row, 3-bit codes
// both halves).  With per-group data types table t of 4-bit codes takes row
// half t & 1 of the region (t >> 1), table t of 3-bit codes region t; so one
// region holds up to two 4-bit tables or one 3-bit table, otherwise two
// regions are needed.  types = 0 means a single codebook.
__host__ __device__ constexpr int table_region_bytes(int bits, int types) {
  return types <= (bits == 4 ? 2 : 1) ? 0x10000 : 0x20000;
}

// Workspace layout of the products (host): every kernel keeps the data that
// must be zero between calls (exchange slots, arrival counters) at the front,
// in [0, workspace_zero_bytes), and leaves them zero; scratch that a call
// may leave as it likes (partial sums) starts at workspace_zero_bytes.  The
// zero region covers every kernel the problem may take, so one workspace
// serves lutq_gemv and lutq_gemm calls of the same problem in any order.
int64_t workspace_zero_bytes(int64_t M, int64_t N, int64_t K);

// Record a device-side error: the first non-zero code wins.
__device__ __forceinline__ void report(int32_t* dev_status, int code) {
  if (dev_status != nullptr) atomicCAS(dev_status, 0, code);
}

// Checked builds (-DLUTQ_BOUNDS): LUTQ_IN_BOUNDS(cond, status) is cond, and a
// false cond is reported as LUTQ_ERR_BOUNDS; the caller skips the access it
// guards.  Other builds: the constant true, so the check and the skip compile
// away.
__device__ __forceinline__ bool bounds_check(bool ok, int32_t* dev_status) {
  if (!ok) report(dev_status, LUTQ_ERR_BOUNDS);
  return ok;
}
#ifdef LUTQ_BOUNDS
#define LUTQ_IN_BOUNDS(cond, status) (::lutq::bounds_check(bool(cond), (status)))
#else
#define LUTQ_IN_BOUNDS(cond, status) (true)
#endif

// Store output value i: fp32, or (y_bf16) the fp32 value rounded once to
// bf16 (round to nearest even; the bf16 output variant of the products).
__device__ __forceinline__ void store_y(float* y, int y_bf16, int64_t i, float v) {
  if (y_bf16) {
    reinterpret_cast<uint16_t*>(y)[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  } else {
    y[i] = v;
  }
}

__device__ __forceinline__ float bf16_lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// 16-byte streaming load that is not kept in L1 (each packed byte is used once).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// One acquire-release atomic add at GPU scope: publishes the calling warp's
// earlier stores (ordered before it by __syncwarp) and, for the caller that
// sees the final count, makes the other contributors' stores visible.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

}  // namespace lutq
