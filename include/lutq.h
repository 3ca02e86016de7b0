/*
 * lutq.h - C ABI of liblutq: group-wise lookup-table (LUT) weight-only
 * quantization and the fused dequantize-and-multiply product, for NVIDIA B200
 * (sm_100a).
 *
 * The operations follow the FLUTE abstract ("Daily Papers" listing, query
 * "group-128"): weights are quantized offline onto a small non-uniform table of
 * levels with one scale per group of 128 weights, the quantized matrix is
 * restructured offline so that unpacking needs few bit operations, and a fused
 * kernel dequantizes on the fly inside the matrix-vector product.
 *
 * Notation: W[N,K] bf16 weights (row n = output feature, K = reduction),
 * G = K/128 groups per row, codebook c[0 .. 2^bits - 1] (bf16), codes
 * q[N,K] (uint8), scales s[N,G] (bf16), x[M,K] bf16 activations, y[M,N] fp32.
 * lutq_pack merges q and s into one packed matrix that the products read.
 * The dequantized weight is s[n, k/128] * c[q[n,k]].
 *
 * Conventions shared by every call:
 *  - All matrices are dense and row-major.  Device pointers must point to
 *    memory of the device that is current on the calling thread, and must be
 *    16-byte aligned (LUTQ_ERR_ALIGN otherwise).
 *  - The caller owns every buffer; the library allocates nothing per call and
 *    keeps no state except a per-device cache of attributes.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL means the legacy default stream).  Argument errors are reported by
 *    the return value before anything is launched.  Conditions found on the
 *    device are written to `*dev_status` (an int32 in device memory, may be
 *    NULL): the kernel stores the lutq_status code there if it was 0, so the
 *    first error wins; the caller reads it after synchronizing.
 *  - Inputs are never modified.
 *  - Shape rules: N % 32 == 0, K % 128 == 0, N >= 32, K >= 128; bits is 3 or 4.
 */
#ifndef LUTQ_H_
#define LUTQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LUTQ_OK = 0,
  LUTQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, unknown enum value */
  LUTQ_ERR_SHAPE = 2,       /* N % 32, K % 128 or M out of the supported range */
  LUTQ_ERR_BITS = 3,        /* bits is not 3 or 4 / does not match the codebook */
  LUTQ_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned */
  LUTQ_ERR_NONFINITE = 5,   /* device: quantize met a NaN or infinite weight */
  LUTQ_ERR_CODE_RANGE = 6,  /* device: pack met a code >= 2^bits, or a typed
                               product a group type without a table */
  LUTQ_ERR_TIMEOUT = 7,     /* device: a bounded wait inside a kernel expired */
  LUTQ_ERR_CUDA = 8,        /* a CUDA runtime call failed */
  LUTQ_ERR_WORKSPACE = 9,   /* workspace missing or smaller than required */
  LUTQ_ERR_BOUNDS = 10      /* device, checked builds only (LUTQ_BUILD_BOUNDS): an
                               index fell outside its buffer; that access was
                               skipped, so the results are unspecified */
} lutq_status;

/*
 * lutq_build_flags - how this library was compiled: a bit mask of
 * LUTQ_BUILD_NVTX (every C-ABI call opens an NVTX range named after the call,
 * for Nsight timelines; compiled with -DLUTQ_NVTX) and LUTQ_BUILD_BOUNDS (the
 * kernels check their global, shared and tensor-memory indices against the
 * buffers' extents and report LUTQ_ERR_BOUNDS through dev_status instead of
 * making the access; compiled with -DLUTQ_BOUNDS, slower, for debugging).
 * The default build returns 0.  No GPU use.
 *
 * No counterpart in the paper: these are tooling options of the library.
 */
#define LUTQ_BUILD_NVTX 1
#define LUTQ_BUILD_BOUNDS 2
int lutq_build_flags(void);

/* Codebook kinds for lutq_codebook. */
typedef enum {
  LUTQ_CODEBOOK_NF4 = 0,        /* 16-level NormalFloat (4 bit) */
  LUTQ_CODEBOOK_LOGB = 1,       /* 16-level logarithmic, base 1.6 (4 bit) */
  LUTQ_CODEBOOK_LLOYD_MAX3 = 2, /* 8-level Lloyd-Max for N(0,1) (3 bit) */
  LUTQ_CODEBOOK_UNIFORM4 = 3    /* 16 evenly spaced levels (4 bit) */
} lutq_codebook_kind;

/* Human-readable name of a status code (static string, never NULL). */
const char* lutq_status_string(int status);

/* Version of the packed layout produced by lutq_pack and read by lutq_gemv /
 * lutq_gemm.  Returns 2 for layout V2 (strips of 32 rows, 16-byte words
 * interleaved across the rows of a strip, then the scales in blocks of 32;
 * see lutq_pack). */
int lutq_layout_version(void);

/* Size in bytes of the packed matrix (codes and scales) of an N x K matrix:
 * N*K/2 + N*K/64 for 4 bits, 3*N*K/8 + N*K/64 for 3 bits.  Returns -1 for
 * an invalid shape or bit width. */
int64_t lutq_packed_bytes(int64_t N, int64_t K, int bits);

/*
 * lutq_codebook - build a codebook on the HOST.
 *
 * Source: the FLUTE abstract (NormalFloat lookup table, 3-bit widths), the
 * Log_bQuant abstract (catalyzex author page: levels spaced in logarithmic
 * space with an adjustable base) and "TurboQuant: A first-principles
 * walkthrough" (the Lloyd-Max algorithm).  Levels are computed in double
 * precision, normalised to max |level| = 1, and rounded once to bf16 (round
 * to nearest even), in ascending order:
 *   NF4: 8 positive and 7 negative standard-normal quantiles plus 0, with the
 *        outermost probability ((1-1/30)+(1-1/32))/2;
 *   LOGB: +-1.6^-k, k = 0..7;
 *   LLOYD_MAX3: the 8-level Lloyd-Max quantizer of N(0,1);
 *   UNIFORM4: (2i-15)/15.
 * out_bf16: host array of (1 << bits) uint16 bf16 bit patterns, written by the
 * call.  Returns LUTQ_ERR_BITS if `bits` does not fit the kind.  No GPU use.
 */
lutq_status lutq_codebook(int kind, int bits, uint16_t* out_bf16);

/*
 * lutq_quantize - group-128 round-to-nearest quantization onto a codebook.
 *
 * Source: the group-128 post-training-quantization study and the FLUTE
 * abstract (both "Daily Papers", query "group-128"): RTN weight-only
 * quantization with one scale per group of 128 consecutive weights along K.
 * For each row n and group g:
 *   s[n,g] = max_{k in g} |W[n,k]|            (exact in bf16)
 *   v      = float(W[n,k]) / float(s[n,g])     (IEEE fp32 divide; 0 if s == 0)
 *   q[n,k] = lowest i minimising the fp32 value |v - c_i|.
 * Subnormal weights are kept (no flush to zero); -0 behaves like +0.
 *
 * W_bf16   device, bf16 [N,K] row-major.
 * codebook device, bf16 [1 << bits], ascending is not required.
 * codes    device, uint8 [N,K] row-major, written.
 * scales   device, bf16 [N,K/128] row-major, written.
 * dev_status device int32 or NULL: LUTQ_ERR_NONFINITE if any weight is NaN or
 *          infinite (codes and scales of that group are then unspecified).
 */
lutq_status lutq_quantize(const void* W_bf16, int64_t N, int64_t K,
                          const void* codebook_bf16, int bits,
                          uint8_t* codes, void* scales_bf16,
                          int32_t* dev_status, void* stream);

/*
 * lutq_quantize_rowscale - lutq_quantize with one scale per row.
 *
 * Source: the Tetra abstract (aiqbench news item) keeps one scale per matrix
 * row; here, without retraining, the row's absolute maximum:
 *   s[n]   = max_k |W[n,k]|                    (exact in bf16)
 *   v      = float(W[n,k]) / float(s[n])       (IEEE fp32 divide; 0 if s == 0)
 *   q[n,k] = lowest i minimising the fp32 value |v - c_i|.
 * s[n] is written to every group's slot of `scales` (bf16 [N,K/128]), so
 * lutq_pack and the products take the result unchanged.  Arguments, errors
 * and asynchrony as lutq_quantize.
 */
lutq_status lutq_quantize_rowscale(const void* W_bf16, int64_t N, int64_t K,
                                   const void* codebook_bf16, int bits, uint8_t* codes,
                                   void* scales_bf16, int32_t* dev_status, void* stream);

/*
 * lutq_quantize_group256 - lutq_quantize with one scale per group of 256
 * consecutive weights along K (the group-size variant of the FLUTE
 * abstract's group quantization): s = max |W| over the 256, v and q as in
 * lutq_quantize.  The scale fills the slots of both 128-groups of `scales`
 * (bf16 [N,K/128]), so lutq_pack and the products take the result unchanged.
 * Returns LUTQ_ERR_SHAPE unless K % 256 == 0; otherwise as lutq_quantize.
 */
lutq_status lutq_quantize_group256(const void* W_bf16, int64_t N, int64_t K,
                                   const void* codebook_bf16, int bits, uint8_t* codes,
                                   void* scales_bf16, int32_t* dev_status, void* stream);

/*
 * lutq_quantize_tensorscale - lutq_quantize with one scale for the matrix.
 *
 * Source: the Log_bQuant abstract (catalyzex author page) compares with
 * asymmetric linear quantization at tensor-wise granularity.  s = max |W|
 * over all of W (exact in bf16), v = float(W[n,k]) / float(s), q as in
 * lutq_quantize; s is written to every slot of `scales`.  With the codebook
 * of lutq_codebook_asym_linear(min W, max W) this is that baseline: levels
 * evenly spaced from min W to max W.  Arguments, errors and asynchrony as
 * lutq_quantize.
 */
lutq_status lutq_quantize_tensorscale(const void* W_bf16, int64_t N, int64_t K,
                                      const void* codebook_bf16, int bits, uint8_t* codes,
                                      void* scales_bf16, int32_t* dev_status, void* stream);

/*
 * lutq_codebook_asym_linear - the asymmetric linear codebook: the 2^bits
 * evenly spaced values from w_min to w_max divided by max(|w_min|, |w_max|),
 * computed in fp64 and rounded once to bf16 (all zero if both are zero).
 * out_bf16: host, 2^bits uint16 bf16 bit patterns, written.  Returns
 * LUTQ_ERR_BITS for bits other than 3 or 4, LUTQ_ERR_INVALID_ARG for a NULL
 * output, non-finite bounds or w_min > w_max.  No GPU use.
 */
lutq_status lutq_codebook_asym_linear(double w_min, double w_max, int bits, uint16_t* out_bf16);

/*
 * lutq_pack - offline restructuring of the codes and scales into layout V2.
 *
 * Source: the FLUTE abstract ("offline restructuring of the quantized weight
 * matrix to minimize bit manipulations associated with unpacking"; 3-bit,
 * non-evenly-divisible widths).
 *
 * Layout V2.  Rows form strips of 32; G = K/128; the unit t = s*G + g is
 * (strip s, group g), U = (N/32)*G units.  The codes of unit t take C bytes
 * at byte t*C, C = 2048 (4 bit) or 1536 (3 bit); its 32 scales take the 64
 * bytes at U*C + t*64.  The codes are 16-byte words; word w of row r (0..31
 * within the strip) is at byte (32*w + r)*16 of the unit's codes, so one word
 * index over a strip is 512 contiguous bytes (one coalesced 16-byte load per
 * lane of a warp).  The scale s[32s + r, g] (bf16 bits, little-endian) is at
 * byte 2*(4*(r % 8) + r / 8) of the unit's 64: the four rows r0, r0+8,
 * r0+16, r0+24 that one lane of the product kernel handles have their
 * scales in 8 consecutive bytes.
 *  4 bit: words 0..3 hold k = 128g + 32w + 0..31; byte i holds the codes
 *         (k0+2i, k0+2i+1), the even one in the low nibble, so every byte is
 *         directly an index into a 256-entry table of code pairs.
 *  3 bit: a code splits into lo2 = q & 3 and hi1 = q >> 2; for a pair (even
 *         e, odd o) lo2(pair) = lo2(e) | lo2(o) << 2, hi2(pair) = hi1(e) |
 *         hi1(o) << 1.  Words 0 and 1 hold k0 = 128g + 64w, pairs P = 0..31;
 *         as four little-endian u32 L_j, byte b has lo2(pair 8j+b) in the low
 *         nibble and lo2(pair 8j+4+b) in the high nibble.  Word 2 is four u32
 *         H_j; byte b holds hi2 of pair 8j+4+b of word 0 (bits 1:0) and of
 *         word 1 (bits 3:2), and hi2 of pair 8j+b of word 0 (bits 5:4) and of
 *         word 1 (bits 7:6).  One AND-OR of L_j with H_j (or H_j >> 2) then
 *         yields four pair indices at once.
 *
 * codes  device, uint8 [N,K] (values < 2^bits).
 * scales device, bf16 [N,K/128] row-major (as lutq_quantize writes them).
 * packed device, lutq_packed_bytes(N,K,bits) bytes, written.
 * dev_status device int32 or NULL: LUTQ_ERR_CODE_RANGE if a code >= 2^bits.
 */
lutq_status lutq_pack(const uint8_t* codes, const void* scales_bf16, int64_t N, int64_t K,
                      int bits, void* packed, int32_t* dev_status, void* stream);

/*
 * lutq_workspace_bytes - device scratch size needed by lutq_gemv / lutq_gemm
 * for this problem, whichever kernel runs it: one 8-byte exchange slot per
 * output value of up to 4 batch rows, where the two halves of a row split
 * between two thread blocks meet (the CUDA-core GEMV), per-tile arrival
 * counters and split-K partial sums (the tensor-core kernel).
 * Returns -1 for an invalid argument.  The value does not depend on the device.
 */
int64_t lutq_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits);

/*
 * lutq_workspace_zero_bytes - the front part of that workspace which every
 * lutq_gemv / lutq_gemm call of this problem finds zero at its start and
 * leaves zero at its end (exchange slots and arrival counters of whichever
 * kernel runs it); the rest is scratch whose contents do not matter.  A
 * workspace therefore needs clearing (e.g. cudaMemset of these bytes) only
 * before its first use.  Returns -1 for an invalid argument.
 */
int64_t lutq_workspace_zero_bytes(int64_t M, int64_t N, int64_t K, int bits);

/*
 * lutq_gemv - fused dequantize-and-multiply for small batches, M = 1..16.
 *
 * Source: the FLUTE abstract (a kernel that fuses dequantization with the
 * matmul; the bottleneck is moving weights from global memory; the lookup
 * table is vectorized and duplicated to ease shared-memory bandwidth) and the
 * BitMoD abstract (the per-group partial sum is rescaled once per group):
 *   y[m,n] = sum_g s[n,g] * ( sum_{k in g} x[m,k] * c[q[n,k]] )
 * Products are bf16 x bf16 (exact in fp32); sums are fp32.  The result is
 * within 2e-3 (relative, floored at 1e-2 of the row's rms) of the exact sum.
 * M = 1..4 run on the CUDA cores (each table lookup serves the M batch rows);
 * larger batches, whose product is a dense contraction for the CUDA cores,
 * and rows whose activations do not fit the kernel's shared memory
 * (M * (K + 2048) > 80896: K above 78848 at M = 1, above 18176 at M = 4) run
 * on the tensor cores exactly as lutq_gemm.  Either way the result does not
 * depend on timing.
 * The CUDA-core kernel is launched as a programmatic dependent of the work
 * before it on `stream`: its set-up overlaps the end of that work, and when
 * its plan leaves multiprocessors free and the packed matrix is at most
 * 64 MiB, extra thread blocks on those multiprocessors
 * bring the matrix into L2 meanwhile.  Nothing is read into the kernel
 * before the preceding work is complete, so the caller need not order
 * anything.
 *
 * x        device bf16 [M,K] row-major.
 * packed   device, layout V2 (lutq_pack): the codes and the scales s.
 * codebook device bf16 [1 << bits].
 * y        device fp32 [M,N] row-major, written (no accumulation into y).
 * workspace device, at least lutq_workspace_bytes(M,N,K,bits) bytes, whose
 *          first lutq_workspace_zero_bytes(M,N,K,bits) bytes are zero-filled
 *          before its first use (e.g. cudaMemset); every call returns the
 *          slots and counters it relies on to zero, so the next call can use
 *          it as it is.  The zero part depends on N only (for M up to
 *          16384), so one workspace serves lutq_gemv and lutq_gemm calls of
 *          any batch size up to the one it was sized for, in any order.
 *          Calls that may run at the same time on the GPU must not share a
 *          workspace.
 * Returns LUTQ_ERR_SHAPE if M is outside 1..16.
 */
lutq_status lutq_gemv(const void* x_bf16, int64_t M, const void* packed,
                      const void* codebook_bf16, int bits, int64_t N, int64_t K, float* y,
                      void* workspace, int64_t workspace_bytes,
                      int32_t* dev_status, void* stream);

/*
 * lutq_gemv_noalloc - lutq_gemv without a caller-provided workspace.
 *
 * No counterpart in the paper: this is a calling convention of the library.
 * It serves callers that cannot allocate device memory where they run the
 * product: code recording CUDA graphs in a capture mode where cudaMalloc is
 * illegal, latency-critical loops that must not call cudaMalloc (it can block
 * and synchronize the device), and plug-in hosts that give a library no
 * allocator.  The scratch that lutq_gemv takes from `workspace` lives here in
 * a fixed library-owned device array of 8 MiB, which every GPU that loads the
 * library holds until the process exits; the call allocates nothing.  The
 * array's first 1 MiB is the zero part of the workspace, the other 7 MiB its
 * scratch.  Arguments other than the workspace, numerics and results are
 * those of lutq_gemv (M = 1..16).
 *  - The first call on a device sets the array up with that device current:
 *    it looks up the array's device address and clears the array with a
 *    synchronous cudaMemset.  Make that first call before any stream capture.
 *  - All calls share the array, which keeps what the last call left: calls
 *    that may overlap on the GPU (other streams, other threads) race and must
 *    be serialized by the caller.  Every call leaves the zero part zero and
 *    no call writes its scratch there, so no call depends on what an earlier
 *    one left (after a call that reported LUTQ_ERR_TIMEOUT the array's
 *    contents, and so later results, are unspecified).
 *  - Returns LUTQ_ERR_WORKSPACE, launching nothing, if
 *    lutq_workspace_zero_bytes(M,N,K,bits) exceeds 1 MiB (N above 32768) or
 *    the scratch of the tensor-core kernel the call may take (4 MiB for
 *    M <= 16) exceeds 7 MiB.
 */
lutq_status lutq_gemv_noalloc(const void* x_bf16, int64_t M, const void* packed,
                              const void* codebook_bf16, int bits, int64_t N, int64_t K,
                              float* y,
                              int32_t* dev_status, void* stream);

/*
 * lutq_gemv_plan - how lutq_gemv divides an N x K problem among thread blocks
 * on a GPU with num_sms multiprocessors (host only; for inspection and tests).
 *
 * No counterpart in the paper: the FLUTE abstract asks for a kernel that
 * keeps every multiprocessor streaming weights; this reports the division
 * that does so.  The packed matrix is a sequence of units (strip of 32 rows,
 * group of 128 codes), strip-major.  plan[6] receives {C, kind, align, Cm, T,
 * nh}: C thread blocks; kind 0 gives block c the units
 * [G*floor(c*S/C), G*floor((c+1)*S/C)) when align = 1 (whole strips) or
 * [floor(c*U/C), floor((c+1)*U/C)) when align = 0 (S = N/32 strips, G = K/128
 * groups, U = S*G units); kind 1 gives block c < Cm groups [0, G-T) of strip
 * c and block Cm + h groups [G-T, G) of strips h*nh .. h*nh+nh-1 (those that
 * exist).  Every strip is then whole in one block or split between two.
 * Returns LUTQ_ERR_SHAPE for N, K as lutq_gemv rejects them,
 * LUTQ_ERR_INVALID_ARG for a NULL plan or num_sms < 1.
 */
lutq_status lutq_gemv_plan(int64_t N, int64_t K, int num_sms, int32_t* plan);

/*
 * lutq_selftest_wait_timeout - checks the bound on the kernels' pipeline waits.
 *
 * No counterpart in the paper: every mbarrier wait inside lutq_gemv and
 * lutq_gemm gives up after a time limit (2 s) and reports LUTQ_ERR_TIMEOUT
 * instead of hanging the GPU.  This call runs that same wait, for limit_ns
 * nanoseconds, on a barrier that nothing completes: afterwards *dev_status
 * (device int32, required) holds LUTQ_ERR_TIMEOUT unless it already held an
 * error, and the stream and context remain usable.  Asynchronous on `stream`.
 * Returns LUTQ_ERR_INVALID_ARG for a NULL dev_status or limit_ns outside
 * 1 .. 1e9.
 */
lutq_status lutq_selftest_wait_timeout(int32_t* dev_status, int64_t limit_ns, void* stream);

/*
 * lutq_selftest_bounds - checks the device-side index checks.
 *
 * No counterpart in the paper.  Runs one kernel that writes a shared array
 * through the kernels' index check with an index one past the extent the
 * check is given (the array itself is larger, so no build makes an access
 * outside memory).  In a build with LUTQ_BUILD_BOUNDS the check skips the
 * write and *dev_status (device int32, required) receives LUTQ_ERR_BOUNDS
 * unless it already held an error; in other builds the check is compiled out
 * and *dev_status is left as it is.  Asynchronous on `stream`.  Returns
 * LUTQ_ERR_INVALID_ARG for a NULL dev_status.
 */
lutq_status lutq_selftest_bounds(int32_t* dev_status, void* stream);

/*
 * lutq_fit_histogram / lutq_fit_codebook - a codebook fitted to a layer.
 *
 * Source: "TurboQuant: A first-principles walkthrough" (the Lloyd-Max
 * algorithm) applied to the layer's own normalised weights, the family of the
 * FLUTE abstract's extension of NormalFloat.  Readings: the data are the
 * values v = fp32(w) / fp32(s) that lutq_quantize compares with the levels
 * (s = the group's absolute maximum, v = 0 for an all-zero group), counted in
 * 16384 bins over [-1, 1]: bin b = floor(fp32(v + 1) * 8192), clamped to
 * 16383, centre c_b = (2b + 1 - 16384) / 16384.  Lloyd-Max from a starting
 * codebook: each bin to its nearest level (fp64 distance, ties to the lower
 * level), each level to the count-weighted mean of its bins' centres (an
 * exact integer ratio; a level with no bins stays), until the assignment
 * repeats or max_iter passes; the levels are rounded once to bf16.
 *
 * lutq_fit_histogram (device): W bf16 [N,K] row-major (K % 128 == 0, N >= 1);
 *   hist device uint64 [16384], ADDED to (zero it first; several matrices
 *   may share one histogram); dev_status: LUTQ_ERR_NONFINITE for a NaN or
 *   infinite weight.  Asynchronous on `stream`; pointers 16-byte aligned.
 * lutq_fit_codebook (HOST, no GPU use): hist host uint64 [16384] (fewer than
 *   2^31 weights in all); init host bf16 [1 << bits] ascending (e.g. from
 *   lutq_codebook); out host bf16 [1 << bits], written (ascending).
 *   Returns LUTQ_ERR_BITS for bits other than 3 or 4, LUTQ_ERR_INVALID_ARG
 *   for NULL pointers, max_iter < 0, a non-finite start or too many counts.
 */
lutq_status lutq_fit_histogram(const void* W_bf16, int64_t N, int64_t K, uint64_t* hist,
                               int32_t* dev_status, void* stream);
lutq_status lutq_fit_codebook(const uint64_t* hist, int bits, const uint16_t* init_bf16,
                              int max_iter, uint16_t* out_bf16);

/*
 * lutq_rht_weights / lutq_rht_activations - randomized Hadamard rotation of
 * every 128-long group of each row.
 *
 * Source: "TurboQuant: A first-principles walkthrough" (a randomized Hadamard
 * transform can replace a uniform random rotation before quantizing).  With H
 * the Sylvester Hadamard matrix of order 128 (H[i][j] = (-1)^popcount(i & j),
 * H H^T = 128 I) and s the caller's 128 random signs:
 *   weights:     g -> H diag(s) g          (offline, before lutq_quantize)
 *   activations: g -> H diag(s) g / 128    (before the product)
 * so that sum_g (H diag(s) w_g) . (H diag(s) x_g / 128) = w . x.  Sums are
 * taken in fp64 and rounded once to bf16 (exact before the rounding for bf16
 * inputs whose exponents span fewer than 38 binades).
 *
 * in       device bf16 [rows, K] row-major (rows = N or M >= 1, K % 128 == 0).
 * signs    device int8 [128]; a negative value means -1, any other +1.
 * out      device bf16 [rows, K], written; may not overlap `in`.
 * Pointers 16-byte aligned.  Asynchronous on `stream`.
 */
lutq_status lutq_rht_weights(const void* W_bf16, int64_t N, int64_t K, const int8_t* signs,
                             void* W_rot_bf16, void* stream);
lutq_status lutq_rht_activations(const void* x_bf16, int64_t M, int64_t K, const int8_t* signs,
                                 void* x_rot_bf16, void* stream);

/*
 * lutq_gemv_rht - lutq_gemv on rotated weights, rotating the activations
 * inside the kernel: y = x_rot . dequant(packed)^T with x_rot the
 * lutq_rht_activations rotation of x (computed on the activations in shared
 * memory, in the kernel's prologue, with the same arithmetic, so the result
 * equals lutq_gemv on lutq_rht_activations(x) bit for bit).  `packed` holds
 * the quantized rotated weights (lutq_rht_weights -> lutq_quantize ->
 * lutq_pack).  Only for products that run on the CUDA-core kernel (M = 1..4
 * and M * (K + 2048) <= 80896); otherwise returns LUTQ_ERR_SHAPE and the
 * caller rotates with lutq_rht_activations and calls lutq_gemm.  Other
 * arguments as lutq_gemv; signs as lutq_rht_activations.
 */
lutq_status lutq_gemv_rht(const void* x_bf16, int64_t M, const void* packed,
                          const void* codebook_bf16, const int8_t* signs, int bits, int64_t N,
                          int64_t K, float* y, void* workspace, int64_t workspace_bytes,
                          int32_t* dev_status, void* stream);

/*
 * lutq_gemv_out_bf16 / lutq_gemm_out_bf16 - lutq_gemv / lutq_gemm writing y as
 * bf16: each fp32 sum that the fp32 calls write is rounded once to bf16
 * (round to nearest even), so y_bf16 equals the fp32 result rounded, bit for
 * bit.  y_bf16: device bf16 [M, N] row-major, 16-byte aligned.  Other
 * arguments, workspace and errors as lutq_gemv / lutq_gemm.
 */
lutq_status lutq_gemv_out_bf16(const void* x_bf16, int64_t M, const void* packed,
                               const void* codebook_bf16, int bits, int64_t N, int64_t K,
                               void* y_bf16, void* workspace, int64_t workspace_bytes,
                               int32_t* dev_status, void* stream);
lutq_status lutq_gemm_out_bf16(const void* x_bf16, int64_t M, const void* packed,
                               const void* codebook_bf16, int bits, int64_t N, int64_t K,
                               void* y_bf16, void* workspace, int64_t workspace_bytes,
                               int32_t* dev_status, void* stream);

/*
 * lutq_gemm - the same product on the tensor cores (tcgen05), for batches
 * where the problem is a dense contraction (tuned for M >= 32; any M >= 1 is
 * accepted).  Arguments and numerics as lutq_gemv.  dev_status receives
 * LUTQ_ERR_TIMEOUT if a pipeline wait inside the kernel exceeds its bound.
 */
lutq_status lutq_gemm(const void* x_bf16, int64_t M, const void* packed,
                      const void* codebook_bf16, int bits, int64_t N, int64_t K, float* y,
                      void* workspace, int64_t workspace_bytes,
                      int32_t* dev_status, void* stream);

/*
 * One scale per group of 64.
 *
 * Source: the group-size variant of the FLUTE abstract's group quantization
 * ("Daily Papers" listing, query "group-128"): the same RTN with a finer
 * group of 64 consecutive weights along K.
 *   s[n,h] = max_{k in h} |W[n,k]|  over the 64-group h (exact in bf16)
 *   v, q   as lutq_quantize.
 *
 * Packed layout: layout V2's code tiles (lutq_pack), then per unit
 * t = strip * (K/128) + g a 128-byte scale block at byte U*C + 128*t (U units,
 * C code bytes per unit): bytes 0..63 hold the scales of the 64-group
 * [128g, 128g + 64), bytes 64..127 those of [128g + 64, 128g + 128), each
 * half in the row order of lutq_pack's 64-byte block (row r at byte
 * 2*(4*(r % 8) + r / 8)).  lutq_packed_bytes_group64 gives the size,
 * U * (C + 128).
 *
 * lutq_quantize_group64: arguments as lutq_quantize; scales_bf16 is
 *   bf16 [N, K/64] row-major, written.
 * lutq_pack_group64: codes uint8 [N,K] and scales bf16 [N, K/64] into a
 *   buffer of lutq_packed_bytes_group64 bytes; errors as lutq_pack.
 * lutq_gemv_group64: y[m,n] = sum_h s[n,h] * sum_{k in h} x[m,k] * c[q[n,k]],
 *   every 64-group's partial sum rescaled once in fp32; M = 1..16, routing,
 *   workspace (lutq_workspace_bytes), numerics and errors as lutq_gemv.
 * lutq_gemm_group64: the same product on the tensor cores (any M >= 1), as
 *   lutq_gemm; each unit's 8 MMAs go to two partials (one per 64-half).
 * All are asynchronous on `stream`; pointers 16-byte aligned.
 */
int64_t lutq_packed_bytes_group64(int64_t N, int64_t K, int bits);
lutq_status lutq_quantize_group64(const void* W_bf16, int64_t N, int64_t K,
                                  const void* codebook_bf16, int bits, uint8_t* codes,
                                  void* scales_bf16, int32_t* dev_status, void* stream);
lutq_status lutq_pack_group64(const uint8_t* codes, const void* scales_bf16, int64_t N,
                              int64_t K, int bits, void* packed, int32_t* dev_status,
                              void* stream);
lutq_status lutq_gemv_group64(const void* x_bf16, int64_t M, const void* packed,
                              const void* codebook_bf16, int bits, int64_t N, int64_t K, float* y,
                              void* workspace, int64_t workspace_bytes, int32_t* dev_status,
                              void* stream);
lutq_status lutq_gemm_group64(const void* x_bf16, int64_t M, const void* packed,
                              const void* codebook_bf16, int bits, int64_t N, int64_t K, float* y,
                              void* workspace, int64_t workspace_bytes, int32_t* dev_status,
                              void* stream);

/*
 * Per-group data types.
 *
 * Source: BitMoD abstract ("Daily Papers" listing, query "group-128"): each
 * group of 128 weights may be quantized with its own numerical data type.
 * Reading (the abstract gives neither the types nor the rule): a layer has T
 * codebooks ("types"), T <= 4 with 4-bit codes and T <= 2 with 3-bit codes
 * (lutq_max_types); every group keeps its absolute-maximum scale, and takes
 * the type whose RTN codes give the smallest squared error
 *   E_t = sum over k = 0, 1, ..., 127 in this order of d_k * d_k,
 *   d_k = fp32(v_k - c_t[q_t[k]]),  v_k = fp32(w_k) / fp32(s),
 * each product exact in fp64 and each addition rounded in fp64; ties go to
 * the lowest type index.  The codes are that type's RTN codes.
 *
 * Packed layout with types: layout V2 (lutq_pack) followed by 8 bytes per
 * unit u = strip * (K / 128) + group at byte U * (C + 64) + 8 u (U units, C
 * code bytes per unit); byte rq (0..7) holds the types of rows rq + 8 i
 * (i = 0..3) of the strip in bits 2i+1:2i.  lutq_packed_bytes_typed gives
 * the size, U * (C + 72).
 *
 * codebooks_bf16  device bf16 [types][2^bits] (type t's levels at t * 2^bits).
 * group_types     device uint8 [N, K/128] row-major.
 *
 * lutq_quantize_typed: as lutq_quantize, and writes group_types.  Returns
 *   LUTQ_ERR_INVALID_ARG for types outside 1..lutq_max_types(bits).
 * lutq_pack_typed: as lutq_pack into a buffer of lutq_packed_bytes_typed
 *   bytes, then the type blocks; dev_status: LUTQ_ERR_CODE_RANGE for a code
 *   >= 2^bits or a type >= lutq_max_types(bits) (stored modulo 4).
 * lutq_gemv_typed: y[m, n] = sum_g s[n, g] * sum_{k in g} x[m, k] *
 *   c_{type[n, g]}[q[n, k]], numerics as lutq_gemv, M = 1..16.  The tables
 *   take 64 KB of shared memory for up to two 4-bit types or one 3-bit type,
 *   128 KB otherwise; the CUDA-core kernel runs M = 1..4 with
 *   M * (K + 2048) <= 80896 (64 KB of tables) or <= 48128 (128 KB), other
 *   products go to the tensor-core kernel (as lutq_gemm_typed).  `types` must
 *   be the count the matrix was quantized with: a group whose stored type is
 *   >= types reads a table that is not filled (unspecified values, no
 *   out-of-bounds access) and the call reports LUTQ_ERR_CODE_RANGE through
 *   dev_status.  Other arguments, workspace and errors as lutq_gemv.
 * lutq_gemm_typed: the same product on the tensor cores (any M >= 1), as
 *   lutq_gemm.
 * All are asynchronous on `stream`; pointers 16-byte aligned.
 */
int lutq_max_types(int bits);
int64_t lutq_packed_bytes_typed(int64_t N, int64_t K, int bits);
lutq_status lutq_quantize_typed(const void* W_bf16, int64_t N, int64_t K,
                                const void* codebooks_bf16, int types, int bits, uint8_t* codes,
                                void* scales_bf16, uint8_t* group_types, int32_t* dev_status,
                                void* stream);
lutq_status lutq_pack_typed(const uint8_t* codes, const void* scales_bf16,
                            const uint8_t* group_types, int64_t N, int64_t K, int bits,
                            void* packed, int32_t* dev_status, void* stream);
lutq_status lutq_gemv_typed(const void* x_bf16, int64_t M, const void* packed,
                            const void* codebooks_bf16, int types, int bits, int64_t N, int64_t K,
                            float* y, void* workspace, int64_t workspace_bytes,
                            int32_t* dev_status, void* stream);
lutq_status lutq_gemm_typed(const void* x_bf16, int64_t M, const void* packed,
                            const void* codebooks_bf16, int types, int bits, int64_t N, int64_t K,
                            float* y, void* workspace, int64_t workspace_bytes,
                            int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LUTQ_H_ */
