// Dequantize-and-multiply on the 5th-generation tensor cores (tcgen05) for
// batches where the product is a dense contraction (the FLUTE abstract,
// "Daily Papers" listing, query "group-128": a kernel that fuses
// dequantization with the matmul; the BitMoD abstract, same listing: the
// per-group partial sum is rescaled once).
//
// Roles of the warps of a CTA (one CTA per SM, persistent; the counts depend
// on the batch tile N_tile, GemmCfg):
//   DW dequantize warps (4 at N_tile >= 64, else 8: two per lane quarter,
//              each taking half of the row's codes; 16 quarter-row warps in
//              the typed 4-bit kernel at N_tile = 16): lane r of warp w owns
//              row 32 (w mod 4) + r of the 128-row tile; it decodes its codes
//              of one group through the lane-duplicated pair table into bf16
//              pairs and stores them into tensor memory (lane = row, column
//              j = codes 2j, 2j+1) as the A operand of the MMA (W is the M
//              side: swap-AB).  The warps load their rows' packed words
//              themselves, straight into registers.
//   4 PG promotion warps (PG = 2 at N_tile = 128, each group owning half of
//              the batch columns): read the group's fp32 partial D[row, batch]
//              from tensor memory, add s[row, g] * partial to registers, and
//              write y (or a split partial) when the row tile's range ends.
//   1 activation warp: loads the activations' 128-wide K slice (two 2-D
//              tensor-map copies, 128-byte swizzle, no multicast).
//   MW MMA warps (2 at N_tile <= 32, taking alternate units; else 1): issue
//              tcgen05.mma kind::f16 (A from tensor memory, B from shared
//              memory, D fp32 in tensor memory), 8 MMAs of K = 16 per group
//              into a fresh partial, and commit to the mbarriers.
// With one scale per group of 64 (G64) each unit has two partials, one per
// 64-half (MMAs 0-3 and 4-7, each into its own partial stage), and the
// promotion warps add s[row, 2g] * first + s[row, 2g + 1] * second.
// Products are exact (bf16 x bf16) and every group's partial is rescaled in
// fp32, so the result matches the fp32-accumulating GEMV up to summation order.
//
// Work split: units (batch tile, row tile, group) in that order; CTA c takes
// units [floor(c U / C), floor((c+1) U / C)).  Row tiles split between CTAs are
// finished per 32-row strip by the last contributor (warp-ordered sums), as
// in the GEMV.  Every mbarrier wait is bounded; on expiry the kernel records
// LUTQ_ERR_TIMEOUT, drains its own copies and MMAs, frees tensor memory and
// returns.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "lutq_common.cuh"
#include "lutq_lut.cuh"
#include "lutq_sm100.cuh"

namespace lutq {

using namespace sm100;

constexpr int kTileRows = 128;
constexpr int kGemmMaxCtas = 256;            // bounds the workspace
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kTmemCols = 512;
template <int NT, bool G64 = false, bool TYPED = false, int BITS = 4>
struct GemmCfg {
  // activation stages (shared memory); two at N_tile = 128 leave 32 KB more
  // to L1 (measured 2% faster at batch 128 than three; four: 25% slower)
  static constexpr int XS = NT >= 128 ? 2 : 4;
  static constexpr int XSTAGE = 2 * NT * 128;       // two boxes of NT rows x 128 bytes
  // A stages in tensor memory (64 columns each) and partial stages (NT
  // columns each).  With one scale per group of 64 a unit fills two partial
  // stages, so the stages go to the partials: at N_tile = 128 two A stages
  // and three partial stages, below it as many partial stages as fit (at
  // most 8).
  // TACC: the typed kernel at N_tile = 128 keeps the promotion warps'
  // running sums in tensor memory (NT columns after the partial stages)
  // instead of registers.  In registers 64 sums a thread spill under the
  // 128-register ceiling of 14 warps, and with the typed kernel's larger
  // table region the spills miss in the L1 that remains (four 4-bit types:
  // 34% slower than the untyped kernel with register sums, 6% with these);
  // the untyped kernel, whose spills stay in L1, is 2% faster with
  // registers.  The sums take two A stages' columns.
  static constexpr bool TACC = TYPED && NT >= 128 && !G64;
  static constexpr int AS = ((G64 || TACC) && NT >= 128) ? 2 : 4;
  static constexpr int DS = G64 ? ((kTmemCols - 64 * AS) / NT < 8 ? (kTmemCols - 64 * AS) / NT : 8)
                                : (NT >= 128 ? 2 : (NT >= 64 ? 3 : 4));
  // dequant warps: 4 (a whole row per lane) at N_tile >= 64; below it 8 (two
  // per lane quarter, half a row each) or, for the typed kernel with 4-bit
  // codes at N_tile = 16, 16 (a quarter of a row each: one 16-byte word per
  // lane and unit).  Measured on the 70B gate/up layer at batch 16: the typed
  // kernel takes 62.0 us with 16 warps against 67.1 us with 8, while the
  // untyped kernel takes 53.4 us with 16 against 50.5 us with 8.  At N_tile
  // = 32 the 23 warps' register share (80) would spill the promotion sums.
  static constexpr int DW = NT >= 64 ? 4 : (TYPED && BITS == 4 && NT <= 16 ? 16 : 8);
  static constexpr int NB = DW >= 8 ? 4 : 2;        // units of packed words in flight per lane
  static constexpr int KC = 64 * 4 / DW;            // A columns written per dequant warp
  static constexpr int PG = NT >= 128 ? 2 : 1;      // promotion warp groups
  static constexpr int NC = NT / PG;                // batch columns per promotion warp
  static constexpr int MW = NT <= 32 ? 2 : 1;      // MMA-issuing warps (see the MMA role)
  static constexpr int WARPS = DW + 4 * PG + 1 + MW;  // dequant, promote, activation load, MMA
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int DCOL = 64 * AS;              // first partial column
  static constexpr int ACOL = DCOL + DS * NT;       // first running-sum column (TACC)
  static_assert(ACOL + (TACC ? NT : 0) <= kTmemCols, "tensor memory columns");
};
constexpr int kMaxPromoteGroups = 2;
constexpr int kScaleRingBytes = 4 * kMaxPromoteGroups * 4 * 32 * 4;  // [warp][SD][lane] u32
// per-group types: the dequant warps' type words travel through a ring of
// asynchronous copies, [warp][NB][lane] u32 (at most 16 warps x 4 units)
constexpr int kTypeRingBytes = 16 * 4 * 32 * 4;

struct GemmArgs {
  const uint8_t* packed;
  const uint8_t* scales;    // the packed matrix's scale blocks (layout V2; 128 bytes per
                            // unit with one scale per group of 64)
  const uint8_t* types;     // per-group data types: the type blocks (else unused)
  const uint16_t* codebook; // [types][2^BITS] with per-group types
  int ntypes;               // tables in `codebook` (1 without per-group types)
  int lut_bytes;            // the table region (table_region_bytes)
  int y_bf16;               // y is bf16 (the fp32 sums rounded once) instead of fp32
  float* y;
  float* part;        // [kGemmMaxCtas][2][4][NT][32]: (CTA, slot, strip, column, row)
  int* counters;      // [BT * NTILES * 4 * kMaxPromoteGroups]
  int32_t* dev_status;
  int64_t N, G, M;
  int64_t ntiles;     // row tiles, ceil(N / 128)
  int64_t U;          // units
  int C;              // CTAs
  int smem_bytes;     // the block's dynamic shared memory (checked builds)
};

// CTA c holds units [g_unit_begin(c), g_unit_begin(c+1)).  The host
// guarantees U * C < 2^32, so the ranges use 32-bit unsigned arithmetic.
__device__ __forceinline__ uint32_t g_unit_begin(uint32_t c, uint32_t U, uint32_t C) {
  return (c * U) / C;
}
__device__ __forceinline__ uint32_t g_unit_owner(uint32_t u, uint32_t U, uint32_t C) {
  return ((u + 1) * C - 1) / U;
}

// Bounded wait used after an abort: only the time limit ends it.
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// Loads chunk_cols<NC>() consecutive columns (32, or 16 when a promotion warp
// owns only 16 columns).
template <int NC>
__host__ __device__ constexpr int chunk_cols() { return NC == 32 ? 32 : 16; }

template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[32]) {
  if (chunk_cols<NC>() == 32) {
    tmem_ld_32x32b_x32(taddr, v);
  } else {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
  }
}

// Write one finished 32-row strip of a row tile for batch tile bt; this warp
// holds batch columns [c0, c0 + NC).
template <int NT, int NC>
__device__ void gemm_finish_strip(const GemmArgs& a, float (&acc)[NC], int64_t seg, int64_t bt,
                                  int64_t row, int sw, int pg, uint32_t u0, int lane) {
  const int c0 = pg * NC;
  const int64_t seg_begin = seg * a.G, seg_end = seg_begin + a.G;
  const int64_t mrem = a.M - bt * kTileRows;
  const int mt = int(mrem < kTileRows ? mrem : kTileRows);
  const uint32_t U = uint32_t(a.U), C = uint32_t(a.C);
  const uint32_t c_lo = g_unit_owner(uint32_t(seg_begin), U, C);
  const uint32_t c_hi = g_unit_owner(uint32_t(seg_end - 1), U, C);
  const int64_t ycol = (bt * kTileRows + c0) * a.N + row;
  const int64_t ysize = a.M * a.N;
  if (c_lo == c_hi) {
#pragma unroll
    for (int j = 0; j < NC; ++j)
      if (c0 + j < mt && LUTQ_IN_BOUNDS(ycol + int64_t(j) * a.N < ysize, a.dev_status))
        store_y(a.y, a.y_bf16, ycol + int64_t(j) * a.N, acc[j]);
    return;
  }
  const int64_t cta = blockIdx.x;
  const int slot = (uint32_t(seg) == uint32_t(u0) / uint32_t(a.G)) ? 0 : 1;
  // checked builds: the partial-sum slot and the counter lie in the workspace
  const int64_t nparts = int64_t(kGemmMaxCtas) * 2 * 4 * NT * 32;
  const int64_t ncounters = ((a.M + kTileRows - 1) / kTileRows) * a.ntiles * 4 * kMaxPromoteGroups;
  const int64_t cidx = (seg * 4 + sw) * kMaxPromoteGroups + pg;
  (void)ysize;  // read by the checks of checked builds only
  (void)nparts;
  (void)ncounters;
  if (!LUTQ_IN_BOUNDS((((cta * 2 + slot) * 4 + sw) * NT + c0 + NC) * 32 <= nparts &&
                          cidx < ncounters,
                      a.dev_status))
    return;
  float* mine = a.part + (((cta * 2 + slot) * 4 + sw) * NT + c0) * 32;
#pragma unroll
  for (int j = 0; j < NC; ++j) mine[j * 32 + lane] = acc[j];
  __syncwarp();
  int arrived = 0;
  int* counter = a.counters + cidx;
  if (lane == 0) arrived = atom_add_acq_rel_gpu(counter, 1);
  arrived = __shfl_sync(0xffffffffu, arrived, 0);
  if (arrived != int(c_hi - c_lo)) return;
  __syncwarp();  // the other lanes' loads follow lane 0's acquire
#pragma unroll
  for (int j = 0; j < NC; ++j) acc[j] = 0.0f;
  for (uint32_t c = c_lo; c <= c_hi; ++c) {
    const int sl = (uint32_t(seg) == g_unit_begin(c, U, C) / uint32_t(a.G)) ? 0 : 1;
    const float* src = a.part + (((c * 2 + sl) * 4 + sw) * NT + c0) * 32;
#pragma unroll
    for (int j = 0; j < NC; ++j) acc[j] += __ldcg(src + j * 32 + lane);
  }
#pragma unroll
  for (int j = 0; j < NC; ++j)
    if (c0 + j < mt && LUTQ_IN_BOUNDS(ycol + int64_t(j) * a.N < ysize, a.dev_status))
      store_y(a.y, a.y_bf16, ycol + int64_t(j) * a.N, acc[j]);
  if (lane == 0) *counter = 0;
}

// Position (batch tile, row tile, group) of consecutive units, advanced
// without divisions.
struct UnitPos {
  uint32_t bt, tau, g;
  __device__ void init(uint32_t u, uint32_t per_bt, uint32_t G) {
    const uint32_t b = u / per_bt, r = u - b * per_bt, t = r / G;
    bt = b;
    tau = t;
    g = r - t * G;
  }
  __device__ void next(int64_t G, int64_t ntiles) {
    if (++g == uint32_t(G)) {
      g = 0;
      if (++tau == uint32_t(ntiles)) {
        tau = 0;
        ++bt;
      }
    }
  }
};

__device__ __forceinline__ void tmem_st_cols32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// Each thread of the warp stores v[0..15] to 16 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_st_cols16(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

template <int BITS, int NT, bool TYPED, bool G64>
__global__ void __launch_bounds__(GemmCfg<NT, G64, TYPED, BITS>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, GemmArgs a) {
  using Cfg = GemmCfg<NT, G64, TYPED, BITS>;
  static_assert(!(TYPED && G64), "per-group types use one scale per group of 128");
  // partials per unit (one per scale), the scale block's bytes
  constexpr int H = G64 ? 2 : 1;
  constexpr int SBB = H * kScaleBytes;
  constexpr int TB = tile_bytes(BITS);
  constexpr int WPR = words_per_row(BITS);
  constexpr int XS = Cfg::XS, AS = Cfg::AS, DS = Cfg::DS, DW = Cfg::DW;
  constexpr int PG = Cfg::PG, NC = Cfg::NC, NB = Cfg::NB;
  constexpr int W_XLOAD = DW + 4 * PG, W_MMA = W_XLOAD + 1;  // MMA warps: W_MMA .. W_MMA + MW - 1
  constexpr int MW = Cfg::MW;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_sa = smem_addr(smem_raw);
  const uint32_t base_sa = (raw_sa + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_sa - raw_sa);
  uint8_t* lut = base;
  const uint32_t lut_sa = base_sa;
  // the table region: 64 KB, or 128 KB for per-group data types that need
  // it (table t of 4-bit codes in row half t & 1 of the 64 KB at (t >> 1)
  // << 16, table t of 3-bit codes in the 64 KB at t << 16, as in the
  // CUDA-core kernel)
  const int LUTB = TYPED ? a.lut_bytes : kLutBytes;
  const uint32_t xst_sa = base_sa + uint32_t(LUTB);
  const uint32_t bar_sa = xst_sa + XS * Cfg::XSTAGE;
  // barrier ids
  constexpr int B_XF = 0, B_XE = XS, B_AF = 2 * XS, B_AE = B_AF + AS, B_DF = B_AE + AS,
                B_DE = B_DF + DS, NBAR = B_DE + DS;
  auto bar = [&](int i) { return bar_sa + 8u * uint32_t(i); };
  uint8_t* misc = base + (bar_sa - base_sa) + 8 * NBAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  uint16_t* cbs = reinterpret_cast<uint16_t*>(misc + 8);
  // checked builds: table, activation stages, barriers, flags, codebook copy
  // and the scale rings lie inside the block's dynamic shared memory
  if (!LUTQ_IN_BOUNDS(bar_sa + 512u + uint32_t(kScaleRingBytes * H) +
                              uint32_t(TYPED ? kTypeRingBytes : 0) - raw_sa <=
                          uint32_t(a.smem_bytes) &&
                          8u * NBAR + 8u + 2u * uint32_t(a.ntypes << BITS) <= 512u,
                      a.dev_status))
    return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < XS; ++i) {
      mbar_init(bar(B_XF + i), 1);
      mbar_init(bar(B_XE + i), 1);
    }
    for (int i = 0; i < AS; ++i) {
      mbar_init(bar(B_AF + i), DW);
      mbar_init(bar(B_AE + i), 1);
    }
    for (int i = 0; i < DS; ++i) {
      mbar_init(bar(B_DF + i), 1);
      mbar_init(bar(B_DE + i), 4 * PG);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (threadIdx.x < (a.ntypes << BITS)) cbs[threadIdx.x] = a.codebook[threadIdx.x];
  if (warp == W_MMA) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  for (int c = threadIdx.x; c < LUTB / 16; c += blockDim.x) {
    // 16-byte chunk c: row e = (c >> 4) & 255, half (c >> 3) & 1 of the
    // 64 KB region c >> 12; without types one table (4-bit codes: both halves)
    const int half = (c >> 3) & 1, region = c >> 12;
    const int t = TYPED ? (BITS == 4 ? 2 * region + half : region) : 0;
    if (t < a.ntypes) {
      const uint32_t v = lut_entry<BITS>(cbs + (t << BITS), (c >> 4) & 255, half);
      reinterpret_cast<uint4*>(lut)[c] = make_uint4(v, v, v, v);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const uint32_t u0 = g_unit_begin(blockIdx.x, uint32_t(a.U), uint32_t(a.C));
  const int n = int(g_unit_begin(blockIdx.x + 1, uint32_t(a.U), uint32_t(a.C)) - u0);
  const uint32_t per_bt = uint32_t(a.ntiles * a.G);

  if (warp < DW) {
    // ---------------------------------------------------------------- dequantize
    // Lane r of warp w loads its row's packed words itself, NB units ahead,
    // straight into registers (16-byte loads, 512 contiguous bytes per warp
    // instruction): a 2 KB bulk copy per strip and unit costs the copy
    // engine about as much as 16 KB of data, and would hold the kernel to
    // about a quarter of the HBM bandwidth.
    const int sw = warp & 3, kh = DW >= 8 ? (warp >> 2) : 0;
    const uint32_t off_e = uint32_t(lane) * 4u, off_o = 128u + uint32_t(lane) * 4u;
    static_assert(DW != 16 || BITS == 4, "quarter rows need 4-bit codes");
    constexpr int NWL = DW == 16 ? 1 : (DW == 8 ? 2 : WPR);  // 16-byte words per lane and unit
    // word j of the lane's words: 4-bit, word kh (DW = 16), words 2kh, 2kh+1
    // (DW = 8) or all; 3-bit, lo word kh and the hi word (DW = 8) or all three
    auto word_of = [&](int j) {
      return DW == 16 ? kh : DW == 8 ? (BITS == 4 ? 2 * kh + j : (j == 0 ? kh : 2)) : j;
    };
    UnitPos fp;  // the next unit to fetch
    fp.init(u0, per_bt, a.G);
    int fetched = 0;
    // per-group types: the lane's row is lane (rq = lane & 7, i = lane >> 3)
    // of its strip; its type is bits 2i+1:2i of byte rq of the unit's block,
    // i.e. bits 8 (lane & 3) + 2i of the block's 4-byte word lane & 4.  That
    // word travels through a ring slot per unit in shared memory (one 4-byte
    // asynchronous copy and one copy group per lane and unit, NB units
    // ahead): a register load per unit beside the code words made the
    // kernel 30% slower at N_tile = 16, even with its value read only at the
    // end.
    const uint32_t ty_ring =
        bar_sa + 512u + uint32_t(kScaleRingBytes * H) + uint32_t(warp * NB * 32 + lane) * 4u;
    auto fetch = [&](uint4 (&wd)[NWL], int slot) {
      if (fetched < n && fp.tau * kTileRows + sw * 32 < a.N &&
          LUTQ_IN_BOUNDS((fp.tau * 4 + sw) * a.G + fp.g < (a.N / kStrip) * a.G, a.dev_status)) {
        const int64_t tile = (fp.tau * 4 + sw) * a.G + fp.g;
        const uint8_t* t = a.packed + tile * TB + lane * 16;
#pragma unroll
        for (int j = 0; j < NWL; ++j) wd[j] = ld_stream_v4(t + word_of(j) * 512);
        if (TYPED)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;"
                       ::"r"(ty_ring + uint32_t(slot * 32 * 4)),
                       "l"(a.types + tile * kTypeBytes + (lane & 4))
                       : "memory");
      }
      if (TYPED) asm volatile("cp.async.commit_group;" ::: "memory");
      ++fetched;
      fp.next(a.G, a.ntiles);
    };
    uint4 ring[NB][NWL];
#pragma unroll
    for (int t = 0; t < NB; ++t) fetch(ring[t], t);
    UnitPos pos;
    pos.init(u0, per_bt, a.G);
    bool ok = true;
    bool bad_type = false;  // a stored type without a table in this call
    // the row's table: 4-bit, type bit 0 -> address bit 7 (row half), bit 1
    // -> bit 16; 3-bit, type bit 0 -> bit 16 (through byte 1 of the column
    // word), masked to the table region, so that a type >= ntypes reads an
    // unfilled table inside it, never the activation stages
    auto sel_of = [&](uint32_t ty) -> uint32_t {
      if (!TYPED) return 0u;
      const uint32_t f = (ty >> (8 * (lane & 3) + 2 * (lane >> 3))) & 3u;
      return (BITS == 4 ? ((f & 1u) << 7) | ((f >> 1) << 8) : (f & 1u) << 8) &
             ((BITS == 4 ? 0x080u : 0u) | (LUTB > kLutBytes ? 0x100u : 0u));
    };
    // decode unit i from wd, refill wd with unit i + NB, hand the tile to the MMA
    auto step = [&](uint4 (&wd)[NWL], int slot, int i) {
      const bool valid = pos.tau * kTileRows + sw * 32 < a.N;
      uint32_t av[32];
      uint32_t ty = 0;
      if (TYPED) {
        // this unit's copy group is complete once at most NB - 1 are pending
        asm volatile("cp.async.wait_group %0;" ::"n"(NB - 1) : "memory");
        ty = lds32(ty_ring + uint32_t(slot * 32 * 4));
      }
      const uint32_t sel = sel_of(ty);
      // a warp that owns the whole row (DW = 4) decodes it in two halves of
      // 32 pairs, storing each before decoding the next (32 registers of
      // pairs live, not 64); the second half's words are kept aside so that
      // the ring slot is refilled right after the first decode, as early as
      // with one half
      uint4 h1[2];
      if (DW == 4) {
        h1[0] = wd[BITS == 4 ? 2 : 1];
        h1[1] = wd[BITS == 4 ? 3 : 2];
      }
      if (valid) {
        // a stored type without a table in this call is reported (once, after the loop)
        if (TYPED)
          bad_type |= ((ty >> (8 * (lane & 3) + 2 * (lane >> 3))) & 3u) >= uint32_t(a.ntypes);
        if (DW == 16) {
          // a quarter row: the 16 pairs of word kh
          const uint32_t v[4] = {wd[0].x, wd[0].y, wd[0].z, wd[0].w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            lookup4(av + 4 * j, v[j], lut_sa, off_e | sel, uint32_t(LUTB), a.dev_status);
        } else {
          const uint4 h0[2] = {wd[0], wd[DW == 8 ? NWL - 1 : (BITS == 4 ? 1 : 2)]};
          decode_group_half<BITS>(av, h0, DW == 8 ? kh : 0, lut_sa, off_e | sel, off_o | sel,
                                  uint32_t(LUTB), a.dev_status);
        }
      }
      fetch(wd, slot);
      const int as = i % AS;
      ok = mbar_wait(bar(B_AE + as), (uint32_t(i / AS) & 1u) ^ 1u, abort_flag, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        return;
      }
      tc_fence_after();
      if (valid) {
        const uint32_t ta =
            tmem + (uint32_t(sw * 32) << 16) + uint32_t(as * 64 + kh * (DW == 16 ? 16 : 32));
        if (DW == 16)
          tmem_st_cols16(ta, av);
        else
          tmem_st_cols32(ta, av);
        if (DW == 4) {
          decode_group_half<BITS>(av, h1, 1, lut_sa, off_e | sel, off_o | sel, uint32_t(LUTB),
                                  a.dev_status);
          tmem_st_cols32(ta + 32u, av);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_AF + as));
      pos.next(a.G, a.ntiles);
    };
    for (int i = 0; i < n && ok; i += NB) {
#pragma unroll
      for (int t = 0; t < NB; ++t) {
        if (i + t >= n || !ok) break;
        step(ring[t], t, i + t);
      }
    }
    if (TYPED) {
      asm volatile("cp.async.wait_all;" ::: "memory");
      if (bad_type) report(a.dev_status, LUTQ_ERR_CODE_RANGE);
    }
  } else if (warp < W_XLOAD) {
    // ---------------------------------------------------------------- promote
    const int sw = warp & 3, pg = (warp - DW) >> 2;
    UnitPos cur;
    cur.init(u0, per_bt, a.G);
    // The group scales of the next SD units travel ahead of use through a
    // ring in shared memory (one 4-byte asynchronous copy per lane, unit and
    // scale, one copy group per unit): waiting for unit i's group never waits for a
    // later unit's load.  Holding the ring in registers and shifting it made
    // every unit wait for the load issued one unit before (a global-load
    // latency per unit).
    constexpr int SD = 4;
    UnitPos pf = cur;
    // ring slot d: H words per lane (its scale of each 64-half with G64)
    const uint32_t ring = bar_sa + 512u + uint32_t((warp - DW) * SD * H * 32 * 4);
    const uint32_t half = uint32_t(scale_slot(lane) >> 1) & 1u;  // which bf16 of the word
    auto issue_scale = [&](const UnitPos& p, int slot, bool live) {
      const int64_t r0 = p.tau * kTileRows + sw * 32;
      if (live && r0 < a.N &&
          LUTQ_IN_BOUNDS((r0 / kStrip) * a.G + p.g < (a.N / kStrip) * a.G, a.dev_status)) {
        const uint8_t* b =
            a.scales + ((r0 / kStrip) * a.G + p.g) * SBB + (scale_slot(lane) & ~3);
#pragma unroll
        for (int h = 0; h < H; ++h)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;"
                       ::"r"(ring + uint32_t(((slot * H + h) * 32 + lane) * 4)),
                       "l"(b + h * kScaleBytes)
                       : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
#pragma unroll
    for (int d = 0; d < SD; ++d) {
      issue_scale(pf, d, d < n);
      pf.next(a.G, a.ntiles);
    }
    float acc[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) acc[j] = 0.0f;
    constexpr int CH = chunk_cols<NC>();
    // TACC: the warp's running sums in tensor memory, its lanes and columns
    // ACOL + pg * NC ..; fresh while the current row tile's range has none
    const uint32_t tacc = tmem + (uint32_t(sw * 32) << 16) + uint32_t(Cfg::ACOL + pg * NC);
    bool fresh = true;
    for (int i = 0; i < n; ++i) {
      const int64_t row = cur.tau * kTileRows + sw * 32 + lane;
      const bool valid = cur.tau * kTileRows + sw * 32 < a.N;
      asm volatile("cp.async.wait_group %0;" ::"n"(SD - 1) : "memory");
      float s[H];
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const uint32_t sw2 = lds32(ring + uint32_t((((i % SD) * H + h) * 32 + lane) * 4));
        s[h] = half ? bf16_hi_to_f32(sw2) : bf16_lo_to_f32(sw2);
      }
      issue_scale(pf, i % SD, i + SD < n);
      pf.next(a.G, a.ntiles);
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const int d = i * H + h, ds = d % DS;  // partial d of the sequence
        const bool ok =
            mbar_wait(bar(B_DF + ds), uint32_t(d / DS) & 1u, abort_flag, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) goto promote_done;
        tc_fence_after();
        const uint32_t tpart = tmem + (uint32_t(sw * 32) << 16) +
                               uint32_t(Cfg::DCOL + ds * NT + pg * NC);
        if (Cfg::TACC) {
          // sum += s * partial, one 32-column chunk at a time; this thread's
          // stores of the previous unit are complete before it reads back
          if (!fresh) tmem_wait_st();
#pragma unroll
          for (int c = 0; c < NC / 32; ++c) {
            uint32_t v[32], u[32];
            tmem_ld_32x32b_x32(tpart + uint32_t(c * 32), v);
            if (!fresh) tmem_ld_32x32b_x32(tacc + uint32_t(c * 32), u);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              u[j] = __float_as_uint(fresh ? s[h] * __uint_as_float(v[j])
                                           : fmaf(s[h], __uint_as_float(v[j]),
                                                  __uint_as_float(u[j])));
            tmem_st_cols32(tacc + uint32_t(c * 32), u);
          }
          fresh = false;
        } else {
#pragma unroll
          for (int c = 0; c < NC / CH; ++c) {
            uint32_t v[32];
            tmem_ld_cols<NC>(tpart + uint32_t(c * CH), v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < CH; ++j)
              acc[c * CH + j] = fmaf(s[h], __uint_as_float(v[j]), acc[c * CH + j]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_DE + ds));
      }
      if (cur.g == a.G - 1 || i == n - 1) {
        if (Cfg::TACC) {
          // the range's sums into registers for the strip's write-out
          tmem_wait_st();
#pragma unroll
          for (int c = 0; c < NC / 32; ++c) {
            uint32_t u[32];
            tmem_ld_32x32b_x32(tacc + uint32_t(c * 32), u);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[c * 32 + j] = __uint_as_float(u[j]);
          }
          fresh = true;
        }
        if (valid)
          gemm_finish_strip<NT, NC>(a, acc, cur.bt * a.ntiles + cur.tau, cur.bt, row, sw, pg, u0,
                                    lane);
#pragma unroll
        for (int j = 0; j < NC; ++j) acc[j] = 0.0f;
      }
      cur.next(a.G, a.ntiles);
    }
  promote_done:
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == W_XLOAD) {
    if (lane == 0) {
      int issued = 0;
      UnitPos pos;
      pos.init(u0, per_bt, a.G);
      for (int i = 0; i < n; ++i, pos.next(a.G, a.ntiles)) {
        const int xs = i % XS;
        if (!mbar_wait(bar(B_XE + xs), (uint32_t(i / XS) & 1u) ^ 1u, abort_flag, kWaitLimitNs))
          break;
        mbar_expect_tx(bar(B_XF + xs), uint32_t(Cfg::XSTAGE));
        const uint32_t xd = xst_sa + uint32_t(xs * Cfg::XSTAGE);
        tma_2d_g2s(xd, &tmap_x, int32_t(pos.g * 128), int32_t(pos.bt * kTileRows), bar(B_XF + xs));
        tma_2d_g2s(xd + NT * 128, &tmap_x, int32_t(pos.g * 128 + 64), int32_t(pos.bt * kTileRows),
                   bar(B_XF + xs));
        issued = i + 1;
      }
      if (*abort_flag) {
        for (int i = (issued > XS ? issued - XS : 0); i < issued; ++i)
          mbar_drain(bar(B_XF + i % XS), uint32_t(i / XS) & 1u);
      }
    }
  } else {
    // ---------------------------------------------------------------- MMA
    // For small batches two warps issue the MMAs, for the even and the odd
    // units: each waits for its unit's operands and stage while the other's
    // MMAs run, so the barrier waits (slow while the table lookups load
    // shared memory) do not leave the tensor pipe idle (16% faster at
    // N_tile = 16; at 64 and above, where each MMA is long, one warp is
    // faster).  Each commits its own MMAs.
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTileRows, NT);
      int issued = -1;  // the last partial d committed
      for (int i = warp - W_MMA; i < n; i += MW) {
        const int xs = i % XS, as = i % AS;
        if (!mbar_wait(bar(B_XF + xs), uint32_t(i / XS) & 1u, abort_flag, kWaitLimitNs)) break;
        if (!mbar_wait(bar(B_AF + as), uint32_t(i / AS) & 1u, abort_flag, kWaitLimitNs)) break;
        const uint32_t xb = xst_sa + uint32_t(xs * Cfg::XSTAGE);
        bool ok = true;
#pragma unroll
        for (int h = 0; h < H; ++h) {
          // partial d = i H + h: MMAs 8h/H .. 8(h+1)/H - 1 of the unit
          const int d = i * H + h, ds = d % DS;
          if (!mbar_wait(bar(B_DE + ds), (uint32_t(d / DS) & 1u) ^ 1u, abort_flag,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = h * (8 / H); kk < (h + 1) * (8 / H); ++kk) {
            const uint32_t b_sa = xb + uint32_t((kk >> 2) * (NT * 128) + (kk & 3) * 32);
            mma_bf16_ts(tmem + uint32_t(Cfg::DCOL + ds * NT), tmem + uint32_t(as * 64 + 8 * kk),
                        smem_desc_k_sw128(b_sa), idesc, kk > h * (8 / H) ? 1u : 0u);
          }
          mma_commit(bar(B_DF + ds));
          issued = d;
        }
        if (!ok) break;
        mma_commit(bar(B_AE + as));
        mma_commit(bar(B_XE + xs));
      }
      if (*abort_flag && issued >= 0) mbar_drain(bar(B_DF + issued % DS), uint32_t(issued / DS) & 1u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) report(a.dev_status, LUTQ_ERR_TIMEOUT);
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------

static int gemm_nt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

// Arrival counters (zero between calls) and split partial sums (scratch).
int64_t gemm_counter_bytes(int64_t M, int64_t N) {
  const int64_t bt = (M + kTileRows - 1) / kTileRows;
  const int64_t ntiles = (N + kTileRows - 1) / kTileRows;
  return (bt * ntiles * 4 * kMaxPromoteGroups * 4 + 255) / 256 * 256;
}
int64_t gemm_scratch_bytes(int64_t M) {
  return int64_t(kGemmMaxCtas) * 2 * 4 * gemm_nt(M) * 32 * 4;
}
int64_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return workspace_zero_bytes(M, N, K) + gemm_scratch_bytes(M);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// x[M, K] bf16 row-major; boxes of 64 (K) x nt (rows), 128-byte swizzle,
// rows past M read as zero.
static cudaError_t make_x_map(CUtensorMap* map, const void* x, int64_t M, int64_t K, int nt) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(M)};
  const cuuint64_t strides[1] = {cuuint64_t(K) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(nt)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int BITS, int NT, bool TYPED, bool G64>
static cudaError_t launch_nt(const CUtensorMap& map, GemmArgs a, int num_sms,
                             cudaStream_t stream) {
  using Cfg = GemmCfg<NT, G64, TYPED, BITS>;
  static int granted[64] = {0};
  // alignment slack, table, activation stages, barriers and flags (512),
  // the promotion warps' scale rings (two scales per lane and unit with G64)
  const int smem = 1024 + a.lut_bytes + Cfg::XS * Cfg::XSTAGE + 512 +
                   kScaleRingBytes * (G64 ? 2 : 1) + (TYPED ? kTypeRingBytes : 0);
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (granted[dev] < smem) {
    err = cudaFuncSetAttribute(gemm_kernel<BITS, NT, TYPED, G64>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    granted[dev] = smem;
  }
  a.C = int(std::min<int64_t>(std::min<int64_t>(num_sms, kGemmMaxCtas), a.U));
  a.smem_bytes = smem;
  gemm_kernel<BITS, NT, TYPED, G64><<<unsigned(a.C), Cfg::THREADS, smem, stream>>>(map, a);
  return cudaGetLastError();
}

template <int BITS, bool TYPED, bool G64 = false>
static cudaError_t launch_nts(int nt, const CUtensorMap& map, const GemmArgs& a, int num_sms,
                              cudaStream_t stream) {
  switch (nt) {
    case 16: return launch_nt<BITS, 16, TYPED, G64>(map, a, num_sms, stream);
    case 32: return launch_nt<BITS, 32, TYPED, G64>(map, a, num_sms, stream);
    case 64: return launch_nt<BITS, 64, TYPED, G64>(map, a, num_sms, stream);
    default: return launch_nt<BITS, 128, TYPED, G64>(map, a, num_sms, stream);
  }
}

// types = 0: one codebook; 1..max_types(bits): per-group data types (the
// packed matrix carries its type blocks and `codebook` holds `types` tables).
// group64: the packed matrix has 128-byte scale blocks (one scale per group
// of 64; types must be 0).
cudaError_t launch_gemm(const void* x, int64_t M, const void* packed, const void* codebook,
                        int bits, int64_t N, int64_t K, float* y, void* workspace,
                        int32_t* dev_status, int num_sms, cudaStream_t stream, int types,
                        bool y_bf16, int64_t zero_bytes, bool group64) {
  const int nt = gemm_nt(M);
  CUtensorMap map;
  std::memset(&map, 0, sizeof(map));
  cudaError_t err = make_x_map(&map, x, M, K, nt);
  if (err != cudaSuccess) return err;
  GemmArgs a;
  a.packed = static_cast<const uint8_t*>(packed);
  a.scales = a.packed + (N / kStrip) * (K / kGroup) * tile_bytes(bits);
  a.types = a.scales + (N / kStrip) * (K / kGroup) * kScaleBytes;
  a.codebook = static_cast<const uint16_t*>(codebook);
  a.ntypes = types > 0 ? types : 1;
  a.lut_bytes = table_region_bytes(bits, types);
  a.y_bf16 = y_bf16 ? 1 : 0;
  a.y = y;
  a.dev_status = dev_status;
  a.N = N;
  a.G = K / kGroup;
  a.M = M;
  a.ntiles = (N + kTileRows - 1) / kTileRows;
  const int64_t bt = (M + kTileRows - 1) / kTileRows;
  a.U = bt * a.ntiles * a.G;
  // unit indices and range arithmetic are 32-bit (U * CTAs < 2^32)
  if (a.U * kGemmMaxCtas >= (int64_t(1) << 32)) return cudaErrorInvalidValue;
  // counters at the front of the workspace, partial sums after its zero region
  if (zero_bytes < 0) zero_bytes = workspace_zero_bytes(M, N, K);
  a.counters = static_cast<int*>(workspace);
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + zero_bytes);
  a.C = 0;
  if (group64) {
    if (types > 0) return cudaErrorInvalidValue;
    return bits == 4 ? launch_nts<4, false, true>(nt, map, a, num_sms, stream)
                     : launch_nts<3, false, true>(nt, map, a, num_sms, stream);
  }
  if (types > 0)
    return bits == 4 ? launch_nts<4, true>(nt, map, a, num_sms, stream)
                     : launch_nts<3, true>(nt, map, a, num_sms, stream);
  return bits == 4 ? launch_nts<4, false>(nt, map, a, num_sms, stream)
                   : launch_nts<3, false>(nt, map, a, num_sms, stream);
}

}  // namespace lutq
