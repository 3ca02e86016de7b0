// Fused dequantize-and-multiply GEMV for batches M = 1..16 on the CUDA cores
// (the FLUTE abstract, "Daily Papers" listing, query "group-128": fuse
// dequantization with the product, duplicate the lookup table against
// shared-memory bandwidth limits; the BitMoD abstract, same listing: rescale
// each group's partial sum once).
//
// Work split.  The packed matrix is a sequence of U = (N/32) * G units, one
// unit = (strip of 32 rows, group of 128 codes) = 2048 (4-bit) or 1536 (3-bit)
// contiguous bytes.  The W active warps of a persistent grid take contiguous,
// equal-length unit ranges [floor(w U / W), floor((w+1) U / W)), so every warp
// streams the same number of bytes.  Inside a unit, lane r owns row 32*strip+r
// and reads its 16-byte words with coalesced 512-byte warp loads.
//
// A strip whose units lie in one warp's range is finished by that warp.  A
// strip split between warps is finished by the last contributor to arrive
// (counted with one atomic per contributor): it adds the contributors'
// partial sums in warp order, so the result does not depend on timing, and
// resets the strip's counter to zero for the next call.
//
// Lookup table.  Each shared-memory row of 256 bytes holds, for one 8-bit
// pair index e, the code pair (c[even], c[odd]) as bf16x2, 32 times for the
// "E" table and 32 times for the "O" table (3-bit only), one copy per lane,
// so a warp-wide lookup never has a bank conflict.  A single byte permute
// turns a packed byte into the lookup address: (byte << 8) | lane offset.
#include "lutq_common.cuh"

namespace lutq {

constexpr int kGemvWarps = 16;                       // warps per CTA
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kLutBytes = 256 * 256;                 // 64 KB
constexpr int kMaxWarpsTotal = 4096;                 // bounds the workspace
constexpr int kXSmemMaxK = 40960;                    // fp32 x staged in shared memory if K <= this

struct GemvArgs {
  const uint16_t* x;        // bf16 [M, K]
  const uint8_t* packed;    // layout V1
  const uint16_t* scales;   // bf16 [N, G]
  const uint16_t* codebook; // bf16 [2^bits]
  float* y;                 // fp32 [M, N]
  float* part;              // [kMaxWarpsTotal][2][M][32] split-strip partial sums
  int* counters;            // [N/32] arrival counters (zero between calls)
  int64_t N, K, G, U;       // U = number of units
  int W;                    // active warps
};

__host__ __device__ inline int64_t unit_begin(int64_t w, int64_t U, int64_t W) { return (w * U) / W; }
// The warp whose range holds unit u.
__host__ __device__ inline int64_t unit_owner(int64_t u, int64_t U, int64_t W) { return ((u + 1) * W - 1) / U; }

__device__ __forceinline__ uint32_t lut_addr(uint32_t word, uint32_t lane_off, int byte) {
  // (byte `byte` of word) << 8 | lane_off  -- lane_off < 256
  return __byte_perm(word, lane_off, 0x5504u | (uint32_t(byte) << 4));
}

__device__ __forceinline__ uint32_t lds32(uint32_t smem_addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(smem_addr));
  return v;
}

__device__ __forceinline__ float4 lds128f(uint32_t smem_addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(smem_addr));
  return v;
}

// acc += (lo, hi) * (x0, x1) elementwise, one packed fp32x2 FMA.
__device__ __forceinline__ void ffma2(float2& acc, float lo, float hi, float x0, float x1) {
  uint64_t a, w, xv;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(acc.x), "f"(acc.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(w) : "f"(lo), "f"(hi));
  asm("mov.b64 %0, {%1, %2};" : "=l"(xv) : "f"(x0), "f"(x1));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a) : "l"(w), "l"(xv));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(acc.x), "=f"(acc.y) : "l"(a));
}

template <int BITS>
__device__ __forceinline__ uint32_t lut_entry(const uint16_t* cb, int e, int half) {
  uint32_t qe, qo;
  if (BITS == 4) {
    qe = e & 15;
    qo = e >> 4;
  } else if (half == 0) {  // E table: lo2 in bits 3:0, hi bits 4 (even) and 5 (odd)
    qe = (e & 3) | (((e >> 4) & 1) << 2);
    qo = ((e >> 2) & 3) | (((e >> 5) & 1) << 2);
  } else {                 // O table: lo2 in bits 7:4, hi bits 0 (even) and 1 (odd)
    qe = ((e >> 4) & 3) | ((e & 1) << 2);
    qo = ((e >> 6) & 3) | (((e >> 1) & 1) << 2);
  }
  return uint32_t(cb[qe]) | (uint32_t(cb[qo]) << 16);
}

// Per-pair multiply-accumulate into the group partial sums.
template <int M, bool XS>
struct PairFma;

template <>
struct PairFma<1, true> {
  // x in shared memory as fp32; one call handles the 4 pairs of one u32
  // index word (8 consecutive k starting at k).
  __device__ __forceinline__ static void run4(float2 (&part)[1], const uint32_t (&lv)[4],
                                              uint32_t xs_addr, int k, const uint16_t*, int64_t) {
    const float4 xa = lds128f(xs_addr + 4u * k);
    const float4 xb = lds128f(xs_addr + 4u * (k + 4));
    ffma2(part[0], bf16_lo_to_f32(lv[0]), bf16_hi_to_f32(lv[0]), xa.x, xa.y);
    ffma2(part[0], bf16_lo_to_f32(lv[1]), bf16_hi_to_f32(lv[1]), xa.z, xa.w);
    ffma2(part[0], bf16_lo_to_f32(lv[2]), bf16_hi_to_f32(lv[2]), xb.x, xb.y);
    ffma2(part[0], bf16_lo_to_f32(lv[3]), bf16_hi_to_f32(lv[3]), xb.z, xb.w);
  }
};

template <int M>
struct PairFma<M, false> {
  // x read from global memory (bf16, L1-cached broadcast loads).
  __device__ __forceinline__ static void run4(float2 (&part)[M], const uint32_t (&lv)[4],
                                              uint32_t, int k, const uint16_t* x, int64_t K) {
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + m * K + k));
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        ffma2(part[m], bf16_lo_to_f32(lv[p]), bf16_hi_to_f32(lv[p]), bf16_lo_to_f32(xw[p]),
              bf16_hi_to_f32(xw[p]));
      }
    }
  }
};

// Decode one 32-bit word of four pair indices into four bf16x2 code pairs.
__device__ __forceinline__ void lookup4(uint32_t (&lv)[4], uint32_t idx, uint32_t lut_base,
                                        uint32_t lane_off) {
#pragma unroll
  for (int b = 0; b < 4; ++b) lv[b] = lds32(lut_base + lut_addr(idx, lane_off, b));
}

template <int BITS, int M, bool XS>
__device__ __forceinline__ void unit_partial(float2 (&part)[M], const uint4 (&wd)[4],
                                             uint32_t lut_base, uint32_t off_e, uint32_t off_o,
                                             uint32_t xs_addr, int kg, const uint16_t* x,
                                             int64_t K) {
  if (BITS == 4) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t v[4] = {wd[w].x, wd[w].y, wd[w].z, wd[w].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t lv[4];
        lookup4(lv, v[j], lut_base, off_e);
        PairFma<M, XS>::run4(part, lv, xs_addr, kg + 32 * w + 8 * j, x, K);
      }
    }
  } else {
    const uint32_t L0[4] = {wd[0].x, wd[0].y, wd[0].z, wd[0].w};
    const uint32_t L1[4] = {wd[1].x, wd[1].y, wd[1].z, wd[1].w};
    const uint32_t H[4] = {wd[2].x, wd[2].y, wd[2].z, wd[2].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t h2 = H[j] >> 2;
      const uint32_t e0 = (L0[j] & 0x0F0F0F0Fu) | (H[j] & 0xF0F0F0F0u);
      const uint32_t o0 = (L0[j] & 0xF0F0F0F0u) | (H[j] & 0x0F0F0F0Fu);
      const uint32_t e1 = (L1[j] & 0x0F0F0F0Fu) | (h2 & 0xF0F0F0F0u);
      const uint32_t o1 = (L1[j] & 0xF0F0F0F0u) | (h2 & 0x0F0F0F0Fu);
      uint32_t lv[4];
      lookup4(lv, e0, lut_base, off_e);
      PairFma<M, XS>::run4(part, lv, xs_addr, kg + 16 * j, x, K);
      lookup4(lv, o0, lut_base, off_o);
      PairFma<M, XS>::run4(part, lv, xs_addr, kg + 16 * j + 8, x, K);
      lookup4(lv, e1, lut_base, off_e);
      PairFma<M, XS>::run4(part, lv, xs_addr, kg + 64 + 16 * j, x, K);
      lookup4(lv, o1, lut_base, off_o);
      PairFma<M, XS>::run4(part, lv, xs_addr, kg + 64 + 16 * j + 8, x, K);
    }
  }
}

template <int BITS>
__device__ __forceinline__ void load_unit(uint4 (&wd)[4], const uint8_t* tile, int lane) {
  constexpr int WPR = words_per_row(BITS);
#pragma unroll
  for (int w = 0; w < WPR; ++w) wd[w] = ld_stream_v4(tile + (32 * w + lane) * kWordBytes);
}

template <int M>
__device__ void finish_strip(const GemvArgs& a, int64_t strip, int64_t warp, int64_t u0, int64_t u1,
                             const float (&acc)[M], int lane) {
  const int64_t row = strip * kStrip + lane;
  const int64_t s_begin = strip * a.G, s_end = s_begin + a.G;
  if (s_begin >= u0 && s_end <= u1) {  // the whole strip is ours
#pragma unroll
    for (int m = 0; m < M; ++m) a.y[m * a.N + row] = acc[m];
    return;
  }
  const int slot = (strip == u0 / a.G) ? 0 : 1;
  float* mine = a.part + ((warp * 2 + slot) * M) * kStrip;
#pragma unroll
  for (int m = 0; m < M; ++m) mine[m * kStrip + lane] = acc[m];
  __threadfence();
  __syncwarp();
  const int64_t w_lo = unit_owner(s_begin, a.U, a.W);
  const int64_t w_hi = unit_owner(s_end - 1, a.U, a.W);
  int arrived = 0;
  if (lane == 0) arrived = atomicAdd(a.counters + strip, 1);
  arrived = __shfl_sync(0xffffffffu, arrived, 0);
  if (arrived != int(w_hi - w_lo)) return;  // not the last contributor
  __threadfence();
  float sum[M];
#pragma unroll
  for (int m = 0; m < M; ++m) sum[m] = 0.0f;
  for (int64_t w = w_lo; w <= w_hi; ++w) {
    const int sl = (strip == unit_begin(w, a.U, a.W) / a.G) ? 0 : 1;
    const float* src = a.part + ((w * 2 + sl) * M) * kStrip;
#pragma unroll
    for (int m = 0; m < M; ++m) sum[m] += __ldcg(src + m * kStrip + lane);
  }
#pragma unroll
  for (int m = 0; m < M; ++m) a.y[m * a.N + row] = sum[m];
  if (lane == 0) a.counters[strip] = 0;
}

template <int BITS, int M, bool XS>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(GemvArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const uint32_t lut_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const uint32_t xs_addr = lut_base + kLutBytes;

  // Build the lane-duplicated pair table: word id -> (entry, half, copy).
  for (int id = threadIdx.x; id < kLutBytes / 4; id += blockDim.x) {
    const int e = id >> 6, half = (id >> 5) & 1;
    reinterpret_cast<uint32_t*>(smem)[id] = lut_entry<BITS>(a.codebook, e, half);
  }
  if (XS) {
    float* xs = reinterpret_cast<float*>(smem + kLutBytes);
    const uint32_t* xw = reinterpret_cast<const uint32_t*>(a.x);
    for (int64_t i = threadIdx.x; i < a.K / 2; i += blockDim.x) {
      const uint32_t v = __ldg(xw + i);
      xs[2 * i] = bf16_lo_to_f32(v);
      xs[2 * i + 1] = bf16_hi_to_f32(v);
    }
  }
  __syncthreads();

  const int64_t warp = int64_t(blockIdx.x) * kGemvWarps + (threadIdx.x >> 5);
  if (warp >= a.W) return;
  const int64_t u0 = unit_begin(warp, a.U, a.W), u1 = unit_begin(warp + 1, a.U, a.W);
  const uint32_t off_e = uint32_t(lane) * 4u, off_o = 128u + uint32_t(lane) * 4u;
  constexpr int TB = tile_bytes(BITS);

  int64_t strip = u0 / a.G;
  int64_t g = u0 - strip * a.G;
  float acc[M];
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = 0.0f;

  uint4 cur[4], nxt[4];
  load_unit<BITS>(cur, a.packed + u0 * TB, lane);
  for (int64_t u = u0; u < u1; ++u) {
    if (u + 1 < u1) load_unit<BITS>(nxt, a.packed + (u + 1) * TB, lane);
    const int64_t row = strip * kStrip + lane;
    const float s = __uint_as_float(uint32_t(a.scales[row * a.G + g]) << 16);
    float2 part[M];
#pragma unroll
    for (int m = 0; m < M; ++m) part[m] = make_float2(0.0f, 0.0f);
    unit_partial<BITS, M, XS>(part, cur, lut_base, off_e, off_o, xs_addr, int(g * kGroup), a.x,
                              a.K);
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = fmaf(s, part[m].x + part[m].y, acc[m]);
    if (g == a.G - 1 || u + 1 == u1) {
      finish_strip<M>(a, strip, warp, u0, u1, acc, lane);
#pragma unroll
      for (int m = 0; m < M; ++m) acc[m] = 0.0f;
      ++strip;
      g = 0;
    } else {
      ++g;
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) cur[w] = nxt[w];
  }
}

int64_t gemv_workspace_bytes(int64_t M, int64_t N) {
  const int64_t counters = ((N / kStrip) * 4 + 255) / 256 * 256;
  return counters + int64_t(kMaxWarpsTotal) * 2 * M * kStrip * 4;
}

// Per device: the largest dynamic shared-memory size already granted to a
// kernel instance, and its resident CTAs per SM at that size.
struct LaunchCache {
  int smem_set[64] = {0};
  int per_sm[64] = {0};
};

template <int BITS, int M, bool XS>
static cudaError_t launch_t(const GemvArgs& a0, int num_sms, cudaStream_t stream) {
  static LaunchCache cache;
  GemvArgs a = a0;
  const int smem = kLutBytes + (XS ? int(a.K) * 4 : 0);
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (cache.smem_set[dev] < smem) {
    err = cudaFuncSetAttribute(gemv_kernel<BITS, M, XS>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    cache.smem_set[dev] = smem;
    cache.per_sm[dev] = 0;
  }
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_kernel<BITS, M, XS>,
                                                      kGemvThreads, smem);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) per_sm = 1;
  int64_t blocks = int64_t(num_sms) * per_sm;
  if (blocks * kGemvWarps > kMaxWarpsTotal) blocks = kMaxWarpsTotal / kGemvWarps;
  const int64_t need = (a.U + kGemvWarps - 1) / kGemvWarps;
  if (blocks > need) blocks = need;
  a.W = int(std::min<int64_t>(blocks * kGemvWarps, a.U));
  gemv_kernel<BITS, M, XS><<<unsigned(blocks), kGemvThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int BITS>
static cudaError_t launch_bits(const GemvArgs& a, int M, int num_sms, cudaStream_t s) {
  const bool xs = a.K <= kXSmemMaxK;
  switch (M) {
    case 1: return xs ? launch_t<BITS, 1, true>(a, num_sms, s) : launch_t<BITS, 1, false>(a, num_sms, s);
    case 2: return launch_t<BITS, 2, false>(a, num_sms, s);
    case 3: return launch_t<BITS, 3, false>(a, num_sms, s);
    case 4: return launch_t<BITS, 4, false>(a, num_sms, s);
    case 5: return launch_t<BITS, 5, false>(a, num_sms, s);
    case 6: return launch_t<BITS, 6, false>(a, num_sms, s);
    case 7: return launch_t<BITS, 7, false>(a, num_sms, s);
    case 8: return launch_t<BITS, 8, false>(a, num_sms, s);
    case 9: return launch_t<BITS, 9, false>(a, num_sms, s);
    case 10: return launch_t<BITS, 10, false>(a, num_sms, s);
    case 11: return launch_t<BITS, 11, false>(a, num_sms, s);
    case 12: return launch_t<BITS, 12, false>(a, num_sms, s);
    case 13: return launch_t<BITS, 13, false>(a, num_sms, s);
    case 14: return launch_t<BITS, 14, false>(a, num_sms, s);
    case 15: return launch_t<BITS, 15, false>(a, num_sms, s);
    case 16: return launch_t<BITS, 16, false>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemv(const void* x, int64_t M, const void* packed, const void* scales,
                        const void* codebook, int bits, int64_t N, int64_t K, float* y,
                        void* workspace, int num_sms, cudaStream_t stream) {
  GemvArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.packed = static_cast<const uint8_t*>(packed);
  a.scales = static_cast<const uint16_t*>(scales);
  a.codebook = static_cast<const uint16_t*>(codebook);
  a.y = y;
  const int64_t counters = ((N / kStrip) * 4 + 255) / 256 * 256;
  a.counters = static_cast<int*>(workspace);
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + counters);
  a.N = N;
  a.K = K;
  a.G = K / kGroup;
  a.U = (N / kStrip) * a.G;
  a.W = 0;
  return bits == 4 ? launch_bits<4>(a, int(M), num_sms, stream)
                   : launch_bits<3>(a, int(M), num_sms, stream);
}

}  // namespace lutq
