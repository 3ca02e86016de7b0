"""CPU oracle for group-wise lookup-table (LUT) weight quantization and the
dequantize-and-multiply product.

TEST INFRASTRUCTURE ONLY.  This is the plain, slow reference that the CUDA
library is checked against.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it.  It shares no code with
the CUDA library and imports nothing from it.

What it follows (web pages, cited by title and section):

* FLUTE abstract ("Daily Papers" listing, query "group-128"): weight-only
  quantization onto a non-uniform lookup table, NormalFloat tables, group size
  128, 3-bit (non-evenly-divisible) widths, and an offline restructuring of the
  quantized matrix so that unpacking needs few bit operations.
* BitMoD abstract (same listing): groups of 128 weights, the per-group partial
  sum rescaled once by the group's scale.
* Group-128 post-training-quantization study (same listing): round-to-nearest
  (RTN) quantization at group size 128.
* Log_bQuant abstract (catalyzex author page): a codebook spaced in
  logarithmic space with an adjustable base.
* "TurboQuant: A first-principles walkthrough": the Lloyd-Max algorithm for an
  optimal scalar quantizer.

The pages print no constants, packing layout or worked example.  Where they are
silent the build's readings are used and stated at each function:

* codebooks are computed in fp64 and rounded once to bf16 (round to nearest
  even); NormalFloat uses the 8-positive / 7-negative / zero quantile
  construction; the log codebook is +-b^-k, k = 0..7, b = 1.6; the 3-bit table is
  the 8-level Lloyd-Max quantizer of N(0,1) normalised to max |level| = 1;
* the group scale is the group's absolute maximum (exact in bf16);
* RTN: v = fp32(w) / fp32(s) (IEEE divide), the code is the lowest index i
  minimising the fp32 value |v - c_i|; an all-zero group uses v = 0;
* the product is y[m, n] = sum_g s[n, g] * sum_{k in g} x[m, k] * c[q[n, k]]
  accumulated in fp64 (every product is exact in fp64).
* per-group types (BitMoD abstract): up to 4 (4-bit) or 2 (3-bit) codebooks;
  a group takes the type of smallest squared RTN error, summed in fp64 in k
  order, lowest index on ties;
* scale variants: one scale per row (Tetra abstract: the row's absolute
  maximum, not retrained), one per matrix with an asymmetric linear codebook
  from min W to max W (the Log_bQuant abstract's baseline), one per 256 or
  per 64 weights along K; the first three fill every 128-group's slot, so
  pack() and gemv() serve them unchanged.

Parity of every function here is pinned in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import math
from typing import Tuple

import numpy as np
import scipy.special

GROUP = 128          # weights per quantization group along K
STRIP = 32           # rows per packing strip (layout V2)
LAYOUT_VERSION = 2

CODEBOOK_KINDS = ("nf4", "logb", "lloyd_max3", "uniform4")


# --------------------------------------------------------------------------
# bf16 helpers
# --------------------------------------------------------------------------

def bf16_round(values) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), once.

    bf16 keeps 8 significant bits.  For a normal value v = m * 2^e with
    m in [1, 2), the result is round_half_even(m * 2^7) * 2^(e-7).
    Returns fp64 values that are exactly representable in bf16.
    """
    v = np.asarray(values, dtype=np.float64)
    out = np.zeros_like(v)
    nz = v != 0.0
    mant, expo = np.frexp(v[nz])            # v = mant * 2^expo, |mant| in [0.5, 1)
    # 8 significant bits: scale |mant| in [0.5,1) by 2^8 -> [128, 256)
    q = np.rint(mant * 256.0)               # numpy rint rounds half to even
    out[nz] = np.ldexp(q, expo - 8)
    return out


def bf16_bits(values) -> np.ndarray:
    """Bit patterns (uint16) of values that are exactly bf16-representable."""
    f32 = np.asarray(values, dtype=np.float64).astype(np.float32)
    if not np.array_equal(f32.astype(np.float64), np.asarray(values, dtype=np.float64)):
        raise ValueError("value not representable in fp32")
    bits = f32.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("value not representable in bf16")
    return (bits >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """uint16 bf16 bit patterns -> float32 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


# --------------------------------------------------------------------------
# Codebooks (fp64), each normalised to max |level| = 1
# --------------------------------------------------------------------------

def nf4_levels() -> np.ndarray:
    """16-level NormalFloat table (FLUTE abstract: "lookup table-based
    NormalFloat quantization").

    Reading: levels are standard-normal quantiles.  A table with an exact zero
    and 16 entries cannot be symmetric, so it takes 8 positive quantiles, 7
    negative ones and 0.  The outermost probability is
    delta = ((1 - 1/30) + (1 - 1/32)) / 2.  Positive levels are Phi^-1(p) for
    the 9 equally spaced p from delta down to 1/2, dropping 1/2; negative levels
    are -Phi^-1(p) for the 8 equally spaced p from delta to 1/2, dropping 1/2.
    The table is sorted and divided by Phi^-1(delta).
    """
    delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))
    p_pos = np.linspace(delta, 0.5, 9)[:-1]
    p_neg = np.linspace(delta, 0.5, 8)[:-1]
    pos = scipy.special.ndtri(p_pos)
    neg = -scipy.special.ndtri(p_neg)
    levels = np.sort(np.concatenate([neg, [0.0], pos]))
    return levels / scipy.special.ndtri(delta)


def logb_levels(base: float = 1.6, per_sign: int = 8) -> np.ndarray:
    """Logarithmic table (Log_bQuant abstract: logarithmic space, adjustable
    base).  Reading: +-base^-k for k = 0 .. per_sign-1, no zero level."""
    mags = base ** (-np.arange(per_sign, dtype=np.float64))
    return np.sort(np.concatenate([-mags, mags]))


def _std_normal_pdf(t):
    return np.exp(-0.5 * np.square(t)) / math.sqrt(2.0 * math.pi)


def _std_normal_mass(a, b):
    """P(a < Z < b) for Z ~ N(0,1), using the tail that avoids cancellation."""
    if a >= 0.0:
        return scipy.special.ndtr(-a) - scipy.special.ndtr(-b)
    return scipy.special.ndtr(b) - scipy.special.ndtr(a)


def lloyd_max_normal(n_levels: int = 8, tol: float = 1e-13,
                     max_iter: int = 100000) -> Tuple[np.ndarray, np.ndarray]:
    """Lloyd-Max quantizer of N(0,1) ("TurboQuant: A first-principles
    walkthrough" names the Lloyd-Max algorithm).

    Alternates the two optimality conditions until the levels move less than
    ``tol``: thresholds are midpoints of adjacent levels; each level is the
    conditional mean of Z over its cell, E[Z | a < Z < b] =
    (pdf(a) - pdf(b)) / P(a < Z < b).  Returns (levels, thresholds), unnormalised.
    """
    y = np.linspace(-2.0, 2.0, n_levels)
    for _ in range(max_iter):
        t = np.concatenate([[-np.inf], 0.5 * (y[:-1] + y[1:]), [np.inf]])
        y_new = np.empty_like(y)
        for i in range(n_levels):
            a, b = t[i], t[i + 1]
            pa = 0.0 if np.isinf(a) else _std_normal_pdf(a)
            pb = 0.0 if np.isinf(b) else _std_normal_pdf(b)
            y_new[i] = (pa - pb) / _std_normal_mass(a, b)
        step = np.max(np.abs(y_new - y))
        y = y_new
        if step < tol:
            break
    t = 0.5 * (y[:-1] + y[1:])
    return y, t


def lloyd_max3_levels() -> np.ndarray:
    """8-level Lloyd-Max table for N(0,1), divided by its largest level."""
    y, _ = lloyd_max_normal(8)
    return y / np.max(np.abs(y))


def uniform4_levels() -> np.ndarray:
    """16 evenly spaced levels (2i - 15) / 15 (a uniform LUT, used by tests)."""
    return (2.0 * np.arange(16) - 15.0) / 15.0


def codebook(kind: str, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """Return (bf16 bit patterns uint16[2^bits], float32 values) for a kind."""
    if kind == "nf4" and bits == 4:
        lv = nf4_levels()
    elif kind == "logb" and bits == 4:
        lv = logb_levels()
    elif kind == "lloyd_max3" and bits == 3:
        lv = lloyd_max3_levels()
    elif kind == "uniform4" and bits == 4:
        lv = uniform4_levels()
    else:
        raise ValueError(f"no codebook {kind!r} with {bits} bits")
    r = bf16_round(lv)
    bits16 = bf16_bits(r)
    return bits16, bf16_bits_to_f32(bits16)


# --------------------------------------------------------------------------
# RTN quantization (group absmax scale, nearest level)
# --------------------------------------------------------------------------

def quantize(w, levels_f32, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """Quantize W[N, K] (values exactly bf16, given as float32) per group of 128.

    s[n, g] = max_{k in g} |W[n, k]|   (a bf16 value, so stored exactly)
    v = fp32(W) / fp32(s)              (IEEE division; 0 when s == 0)
    q = lowest i minimising fp32 |v - c_i|, scanning i = 0 .. 2^bits - 1 and
        replacing the best only on a strictly smaller distance.

    Returns (codes uint8[N, K], scale bf16 bit patterns uint16[N, K/128]).
    Raises ValueError on non-finite weights.
    """
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    levels = np.asarray(levels_f32, dtype=np.float32)
    if levels.shape != (1 << bits,):
        raise ValueError("codebook size must be 2^bits")
    g = k // GROUP
    wg = w.reshape(n, g, GROUP)
    s = np.max(np.abs(wg), axis=2)                          # float32, exact
    s_b = np.broadcast_to(s[:, :, None], wg.shape)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s_b > 0, wg / s_b, np.float32(0.0)).astype(np.float32)
    best_d = np.full(v.shape, np.inf, dtype=np.float32)
    best_i = np.zeros(v.shape, dtype=np.uint8)
    for i in range(levels.size):
        d = np.abs(v - levels[i])                           # float32 subtract
        take = d < best_d
        best_i[take] = i
        best_d[take] = d[take]
    scale_bits = (s.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return best_i.reshape(n, k), scale_bits


def quantize_rowscale(w, levels_f32, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """RTN with one scale per row (Tetra abstract, aiqbench news item: one
    scale per matrix row; here the row's absolute maximum, not retrained).

    s[n] = max_k |W[n, k]|; v = fp32(W) / fp32(s[n]) (0 when s == 0); q as in
    quantize().  The scale is returned in every group's slot, scale bits
    uint16[N, K/128], so packing and the product are those of quantize().
    """
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    levels = np.asarray(levels_f32, dtype=np.float32)
    if levels.shape != (1 << bits,):
        raise ValueError("codebook size must be 2^bits")
    s = np.max(np.abs(w), axis=1)                            # float32, exact
    s_b = np.broadcast_to(s[:, None], w.shape)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s_b > 0, w / s_b, np.float32(0.0)).astype(np.float32)
    best_d = np.full(v.shape, np.inf, dtype=np.float32)
    best_i = np.zeros(v.shape, dtype=np.uint8)
    for i in range(levels.size):
        d = np.abs(v - levels[i])
        take = d < best_d
        best_i[take] = i
        best_d[take] = d[take]
    sb_row = (s.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return best_i, np.repeat(sb_row[:, None], k // GROUP, axis=1)


def quantize_group256(w, levels_f32, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """RTN with one scale per group of 256 along K (the group-size variant):
    s = max |W| over the 256 weights, v = fp32(W) / fp32(s), q as in
    quantize(); each 256-group's scale fills the slots of its two 128-groups,
    so packing and the product are those of quantize().  K % 256 == 0."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    if k % 256:
        raise ValueError("K must be a multiple of 256")
    codes, sb = quantize_rowscale(w.reshape(n * (k // 256), 256), levels_f32, bits)
    return codes.reshape(n, k), np.repeat(sb[:, 0].reshape(n, k // 256), 2, axis=1)


def quantize_group64(w, levels_f32, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """RTN with one scale per group of 64 along K (the finer group-size
    variant): s = max |W| over the 64, v and q as in quantize().  Returns
    (codes uint8[N, K], scale bits uint16[N, K/64])."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    levels = np.asarray(levels_f32, dtype=np.float32)
    if levels.shape != (1 << bits,):
        raise ValueError("codebook size must be 2^bits")
    wg = w.reshape(n, k // 64, 64)
    s = np.max(np.abs(wg), axis=2)
    s_b = np.broadcast_to(s[:, :, None], wg.shape)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s_b > 0, wg / s_b, np.float32(0.0)).astype(np.float32)
    best_d = np.full(v.shape, np.inf, dtype=np.float32)
    best_i = np.zeros(v.shape, dtype=np.uint8)
    for i in range(levels.size):
        d = np.abs(v - levels[i])
        take = d < best_d
        best_i[take] = i
        best_d[take] = d[take]
    return best_i.reshape(n, k), (s.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def pack_group64(codes, scale_bits, bits: int) -> np.ndarray:
    """Layout V2 with 128-byte scale blocks: the codes as pack(); then for
    unit t = s * G + g the 128 bytes at U * C + 128 t, the first 64 holding
    the scales of the 64-group k in [128 g, 128 g + 64) and the second 64 those
    of [128 g + 64, 128 g + 128), each half in the row order of pack()'s
    64-byte block (row r at byte 2 * (4 * (r % 8) + r // 8))."""
    q = np.asarray(codes, dtype=np.uint8)
    n, k = q.shape
    _check_shape(n, k)
    sb = np.asarray(scale_bits, dtype=np.uint16)
    if sb.shape != (n, k // 64):
        raise ValueError("scales shape mismatch")
    code_tiles = _pack_codes(q, bits)
    ns, g = n // STRIP, k // GROUP
    sc = sb.reshape(ns, 4, 8, g, 2).transpose(0, 3, 4, 2, 1)    # [s, g, half, rq, i]
    sc_bytes = np.ascontiguousarray(sc).astype("<u2").view(np.uint8).reshape(-1)
    return np.concatenate([code_tiles.reshape(-1), sc_bytes])


def gemv_group64(x, codes, scale_bits, levels_f32) -> np.ndarray:
    """y[m, n] = sum_h s[n, h] * sum_{k in h} x[m, k] * c[q[n, k]] over the
    64-groups h, in fp64."""
    xf = np.asarray(x, dtype=np.float64)
    q = np.asarray(codes)
    n, k = q.shape
    m = xf.shape[0]
    h = k // 64
    c = np.asarray(levels_f32, dtype=np.float64)
    cq = c[q].reshape(n, h, 64)
    s = bf16_bits_to_f32(scale_bits).astype(np.float64)
    partial = np.einsum("mhk,nhk->hmn", xf.reshape(m, h, 64), cq)
    return np.sum(partial * s.T[:, None, :], axis=0)


def quantize_tensorscale(w, levels_f32, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """RTN with one scale for the whole matrix (tensor-wise granularity, the
    comparison baseline of the Log_bQuant abstract): s = max |W| over all
    entries, v = fp32(W) / fp32(s), q as in quantize(); s in every slot."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    codes, sb = quantize_rowscale(np.concatenate([w.reshape(1, -1)]), levels_f32, bits)
    return codes.reshape(n, k), np.full((n, k // GROUP), sb[0, 0], dtype=np.uint16)


def asym_linear_levels(w_min: float, w_max: float, bits: int) -> np.ndarray:
    """Asymmetric linear codebook (Log_bQuant abstract: asymmetric linear
    quantization, the uniform baseline it compares with).  Reading: the 2^bits
    evenly spaced values from w_min to w_max, divided by S = max(|w_min|,
    |w_max|) so that they lie in [-1, 1] (the matrix's scale S then comes from
    quantize_tensorscale); computed in fp64, rounded once to bf16."""
    if not (w_min <= w_max) or not np.isfinite(w_min) or not np.isfinite(w_max):
        raise ValueError("need finite w_min <= w_max")
    s = max(abs(w_min), abs(w_max))
    n = 1 << bits
    if s == 0:
        return np.zeros(n)
    i = np.arange(n, dtype=np.float64)
    return bf16_round((w_min + i * (w_max - w_min) / (n - 1)) / s)


# --------------------------------------------------------------------------
# Packing, layout V2 (the offline restructuring of the FLUTE abstract)
# --------------------------------------------------------------------------
#
# Rows come in strips of 32; groups are 128 codes along K.  Unit t = s * G + g
# is (strip s, group g); there are U = (N / 32) * G units.  The codes of unit
# t take C bytes at byte t * C, C = 2048 (4-bit) or 1536 (3-bit); its 32
# scales take the 64 bytes at U * C + t * 64.  The codes are a sequence of
# 16-byte words; word w of row r (r in 0..31 within the strip) sits at byte
# (32 * w + r) * 16 of the unit's codes, so one word index over a strip is 512
# contiguous bytes.  The scale of row r (bf16 bits, little-endian) sits at
# byte 2 * (4 * (r % 8) + r // 8) of the unit's 64.
#
# 4-bit: words w = 0..3 cover k = 128g + 32w + (0..31).  Byte i of the word
#   holds the pair of codes (k0 + 2i, k0 + 2i + 1): even code in the low nibble.
# 3-bit: a code q is split into lo2 = q & 3 and hi1 = q >> 2.  For a pair of
#   codes (even e, odd o): lo2(pair) = lo2(e) | lo2(o) << 2 and
#   hi2(pair) = hi1(e) | hi1(o) << 1.
#   Words 0 and 1 ("lo planes") cover k0 = 128g + 64w, i.e. 32 pairs
#   P = 0..31 with pair P = codes (k0 + 2P, k0 + 2P + 1).  Read as four
#   little-endian u32 L_j (j = 0..3), byte b of L_j holds lo2(pair 8j + b) in
#   its low nibble and lo2(pair 8j + 4 + b) in its high nibble.
#   Word 2 ("hi plane") is four u32 H_j; byte b of H_j holds
#     bits 1:0 = hi2(pair 8j + 4 + b of lo word 0)
#     bits 3:2 = hi2(pair 8j + 4 + b of lo word 1)
#     bits 5:4 = hi2(pair 8j + b     of lo word 0)
#     bits 7:6 = hi2(pair 8j + b     of lo word 1)

SCALE_BLOCK = 64     # bytes of one unit's scales


def code_bytes(bits: int) -> int:
    """Bytes of codes of one unit."""
    if bits == 4:
        return 2048
    if bits == 3:
        return 1536
    raise ValueError("bits must be 3 or 4")


def packed_bytes(n: int, k: int, bits: int) -> int:
    return (n // STRIP) * (k // GROUP) * (code_bytes(bits) + SCALE_BLOCK)


def _check_shape(n: int, k: int) -> None:
    if n % STRIP or k % GROUP:
        raise ValueError("N must be a multiple of 32 and K of 128")


def pack(codes, scale_bits, bits: int) -> np.ndarray:
    """codes uint8[N, K] and scale_bits uint16[N, K/128] (bf16 bits) ->
    packed uint8[packed_bytes(N, K, bits)] (layout V2)."""
    q = np.asarray(codes, dtype=np.uint8)
    n, k = q.shape
    _check_shape(n, k)
    sb = np.asarray(scale_bits, dtype=np.uint16)
    if sb.shape != (n, k // GROUP):
        raise ValueError("scales shape mismatch")
    code_tiles = _pack_codes(q, bits)                       # [s, g, C]
    ns, g = n // STRIP, k // GROUP
    # row r = 8 i + rq of strip s -> scale position 4 rq + i
    sc = sb.reshape(ns, 4, 8, g).transpose(0, 3, 2, 1)      # [s, g, rq, i]
    sc_bytes = np.ascontiguousarray(sc).astype("<u2").view(np.uint8).reshape(-1)
    return np.concatenate([code_tiles.reshape(-1), sc_bytes])


def _pack_codes(q, bits: int) -> np.ndarray:
    """The code bytes of every tile, [strips, groups, code_bytes(bits)]."""
    n, k = q.shape
    if np.any(q >= (1 << bits)):
        raise ValueError("code out of range")
    ns, g = n // STRIP, k // GROUP
    if bits == 4:
        # index order of a code: row = 32 s + r, k = 128 g + 32 w + 2 i + e
        t = q.reshape(ns, STRIP, g, 4, 16, 2)
        byte = t[..., 0] | (t[..., 1] << 4)                 # [s, r, g, w, i]
        tiles = byte.transpose(0, 2, 3, 1, 4)               # [s, g, w, r, i]
        return np.ascontiguousarray(tiles).reshape(ns, g, -1)
    if bits == 3:
        # k = 128 g + 64 w + 16 j + 8 h + 2 b + e  (h: low/high nibble half)
        t = q.reshape(ns, STRIP, g, 2, 4, 2, 4, 2)
        even, odd = t[..., 0], t[..., 1]                    # [s, r, g, w, j, h, b]
        lo2 = (even & 3) | ((odd & 3) << 2)
        hi2 = (even >> 2) | ((odd >> 2) << 1)
        lo_byte = lo2[:, :, :, :, :, 0, :] | (lo2[:, :, :, :, :, 1, :] << 4)  # [s,r,g,w,j,b]
        hi_byte = (hi2[:, :, :, 0, :, 1, :]
                   | (hi2[:, :, :, 1, :, 1, :] << 2)
                   | (hi2[:, :, :, 0, :, 0, :] << 4)
                   | (hi2[:, :, :, 1, :, 0, :] << 6))                          # [s,r,g,j,b]
        lo_words = lo_byte.reshape(ns, STRIP, g, 2, 16)     # byte 4j + b of word w
        hi_words = hi_byte.reshape(ns, STRIP, g, 1, 16)
        words = np.concatenate([lo_words, hi_words], axis=3)  # [s, r, g, 3, 16]
        tiles = words.transpose(0, 2, 3, 1, 4)              # [s, g, w, r, 16]
        return np.ascontiguousarray(tiles).reshape(ns, g, -1).astype(np.uint8)
    raise ValueError("bits must be 3 or 4")


def unpack(packed, n: int, k: int, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """Inverse of :func:`pack`, written byte by byte from the layout text:
    (codes uint8[N, K], scale_bits uint16[N, K/128])."""
    p = np.asarray(packed, dtype=np.uint8)
    _check_shape(n, k)
    if p.size != packed_bytes(n, k, bits):
        raise ValueError("packed size mismatch")
    g = k // GROUP
    q = np.zeros((n, k), dtype=np.uint8)
    sb = np.zeros((n, g), dtype=np.uint16)
    cb = code_bytes(bits)
    units = (n // STRIP) * g
    for row in range(n):
        s, r = divmod(row, STRIP)
        for gi in range(g):
            t = s * g + gi
            base = t * cb
            at = units * cb + t * SCALE_BLOCK + 2 * (4 * (r % 8) + r // 8)
            sb[row, gi] = int(p[at]) | (int(p[at + 1]) << 8)
            if bits == 4:
                for w in range(4):
                    word = p[base + (32 * w + r) * 16: base + (32 * w + r) * 16 + 16]
                    for i in range(16):
                        kk = GROUP * gi + 32 * w + 2 * i
                        q[row, kk] = word[i] & 15
                        q[row, kk + 1] = word[i] >> 4
            else:
                lo = [p[base + (32 * w + r) * 16: base + (32 * w + r) * 16 + 16] for w in (0, 1)]
                hi = p[base + (64 + r) * 16: base + (64 + r) * 16 + 16]
                for w in (0, 1):
                    for j in range(4):
                        for b in range(4):
                            byte_lo = int(lo[w][4 * j + b])
                            byte_hi = int(hi[4 * j + b])
                            for h in (0, 1):
                                pair = 8 * j + 4 * h + b
                                l2 = (byte_lo >> (4 * h)) & 15
                                shift = (2 * w) if h == 1 else (4 + 2 * w)
                                h2 = (byte_hi >> shift) & 3
                                kk = GROUP * gi + 64 * w + 2 * pair
                                q[row, kk] = (l2 & 3) | ((h2 & 1) << 2)
                                q[row, kk + 1] = ((l2 >> 2) & 3) | (((h2 >> 1) & 1) << 2)
    return q, sb


# --------------------------------------------------------------------------
# Dequantization and the product
# --------------------------------------------------------------------------

def dequant(codes, scale_bits, levels_f32) -> np.ndarray:
    """W_hat[n, k] = s[n, k/128] * c[q[n, k]] in fp64 (exact: 8-bit x 8-bit
    significands)."""
    q = np.asarray(codes)
    s = bf16_bits_to_f32(scale_bits).astype(np.float64)
    c = np.asarray(levels_f32, dtype=np.float64)
    n, k = q.shape
    return (c[q].reshape(n, k // GROUP, GROUP) * s[:, :, None]).reshape(n, k)


def gemv(x, codes, scale_bits, levels_f32) -> np.ndarray:
    """y[m, n] = sum_g s[n, g] * (sum_{k in g} x[m, k] * c[q[n, k]]), fp64.

    The inner sum is the per-group partial sum and the scale is applied once
    per group (BitMoD abstract: rescale the per-group partial sum).
    x is float32 (bf16-valued) [M, K]; returns float64 [M, N].
    """
    xf = np.asarray(x, dtype=np.float64)
    q = np.asarray(codes)
    n, k = q.shape
    m = xf.shape[0]
    g = k // GROUP
    c = np.asarray(levels_f32, dtype=np.float64)
    s = bf16_bits_to_f32(scale_bits).astype(np.float64)       # [N, G]
    cq = c[q].reshape(n, g, GROUP).transpose(1, 2, 0)         # [G, 128, N]
    xg = xf.reshape(m, g, GROUP).transpose(1, 0, 2)           # [G, M, 128]
    partial = np.matmul(xg, cq)                                # [G, M, N]
    return np.sum(partial * s.T[:, None, :], axis=0)


# --------------------------------------------------------------------------
# Randomized Hadamard rotation ("TurboQuant: A first-principles walkthrough":
# before quantizing, a randomized Hadamard transform can stand in for a
# uniform random rotation)
# --------------------------------------------------------------------------
#
# Readings (the page gives no construction): the rotation acts on each group
# of 128 consecutive k; it is R = H diag(s) with H the Sylvester Hadamard
# matrix of order 128 (entries +-1, H H^T = 128 I) and s a vector of 128
# random signs that the caller draws and passes in.  The weights are rotated
# offline without normalisation, w_g -> H diag(s) w_g (exact integer
# combinations of the bf16 weights, rounded once to bf16), and the
# activations online with the 1/128 that makes the pair orthogonal,
# x_g -> H diag(s) x_g / 128 (rounded once to bf16).  Then
# sum_g (R w_g) . (R x_g) / 128 = sum_g w_g . x_g.

def hadamard(n: int = GROUP) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (a power of two), by the doubling
    recursion H_2m = [[H_m, H_m], [H_m, -H_m]]."""
    if n < 1 or n & (n - 1):
        raise ValueError("order must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def _check_signs(signs) -> np.ndarray:
    s = np.asarray(signs, dtype=np.float64).reshape(-1)
    if s.size != GROUP or not np.all(np.abs(s) == 1.0):
        raise ValueError("signs must be 128 values of +1 or -1")
    return s


def rht_weights(w, signs) -> np.ndarray:
    """W[N, K] -> each row's groups w_g replaced by H diag(s) w_g, computed in
    fp64 and rounded once to bf16 (returned as fp64 values)."""
    s = _check_signs(signs)
    wf = np.asarray(w, dtype=np.float64)
    n, k = wf.shape
    _check_shape(STRIP, k)
    h = hadamard(GROUP)
    rot = np.matmul(wf.reshape(n, k // GROUP, GROUP) * s, h.T)   # row vectors: (H v)^T = v^T H^T
    return bf16_round(rot.reshape(n, k))


def rht_activations(x, signs) -> np.ndarray:
    """x[M, K] -> each row's groups x_g replaced by H diag(s) x_g / 128, fp64,
    rounded once to bf16 (returned as fp64 values)."""
    s = _check_signs(signs)
    xf = np.asarray(x, dtype=np.float64)
    m, k = xf.shape
    _check_shape(STRIP, k)
    h = hadamard(GROUP)
    rot = np.matmul(xf.reshape(m, k // GROUP, GROUP) * s, h.T) / GROUP
    return bf16_round(rot.reshape(m, k))


# --------------------------------------------------------------------------
# Codebook fitted to a layer (Lloyd-Max on the layer's own normalised
# weights: "TurboQuant: A first-principles walkthrough" names the Lloyd-Max
# algorithm; the FLUTE abstract speaks of extending NormalFloat)
# --------------------------------------------------------------------------
#
# Readings (the pages give no procedure): the data are the normalised weights
# v = fp32(w) / fp32(s) of the quantizer (s = the group's absolute maximum);
# they are counted in HIST_BINS equal bins over [-1, 1], bin
# b = floor(fp32(v + 1) * HIST_BINS / 2) (clamped to the last bin), whose
# centre is c_b = (2 b + 1 - HIST_BINS) / HIST_BINS; Lloyd-Max then alternates
# (1) each bin to its nearest level (fp64 distance, ties to the lowest level)
# and (2) each level to the count-weighted mean of its bins' centres, an exact
# integer ratio (a level whose cell is empty stays), from a starting codebook
# until the assignment no longer changes or max_iter passes; the levels are
# rounded once to bf16.

HIST_BINS = 16384


def fit_histogram(w) -> np.ndarray:
    """Counts (int64[HIST_BINS]) of W's normalised weights v = w / s."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    wg = w.reshape(n, k // GROUP, GROUP)
    s = np.broadcast_to(np.max(np.abs(wg), axis=2)[:, :, None], wg.shape)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s > 0, wg / s, np.float32(0.0)).astype(np.float32)
    b = np.floor((v + np.float32(1.0)).astype(np.float32) * np.float32(HIST_BINS // 2))
    b = np.minimum(b.astype(np.int64), HIST_BINS - 1)
    return np.bincount(b.reshape(-1), minlength=HIST_BINS).astype(np.int64)


def fit_codebook(hist, init_levels, max_iter: int = 100) -> np.ndarray:
    """Lloyd-Max on a fit_histogram histogram from init_levels (ascending);
    returns the levels rounded to bf16 (fp64 values)."""
    counts = np.asarray(hist, dtype=np.int64).reshape(-1)
    if counts.size != HIST_BINS:
        raise ValueError("histogram size")
    levels = np.asarray(init_levels, dtype=np.float64).copy()
    ints = 2 * np.arange(HIST_BINS, dtype=np.int64) + 1 - HIST_BINS   # centre * HIST_BINS
    centres = ints / float(HIST_BINS)                                  # exact in fp64
    assign = None
    for _ in range(max_iter):
        # nearest level in fp64; argmin keeps the first (lowest) of equal distances
        new_assign = np.argmin(np.abs(centres[:, None] - levels[None, :]), axis=1)
        if assign is not None and np.array_equal(new_assign, assign):
            break
        assign = new_assign
        for i in range(levels.size):
            cell = assign == i
            den = int(np.sum(counts[cell]))
            if den:
                num = int(np.sum(counts[cell] * ints[cell]))   # exact: |num| < 2^59
                levels[i] = float(num) / float(den * HIST_BINS)
    return bf16_round(levels)


# --------------------------------------------------------------------------
# Per-group data types (BitMoD abstract: each group of 128 weights may be
# quantized with its own numerical data type)
# --------------------------------------------------------------------------
#
# Readings (the abstract names the idea, not the types or the rule): a layer
# has T codebooks ("types"), T <= 4 for 4-bit codes and T <= 2 for 3-bit
# codes.  Every group keeps the absolute-maximum scale s; for each type t the
# codes q_t are the RTN codes of quantize() on that type's levels, and the
# group's error is
#     E_t = sum over k = 0, 1, ..., 127 in this order of d_k * d_k,
#     d_k = fp32(v_k - c_t[q_t[k]])   (the RTN distance, signed),
# each product exact in fp64 and each addition rounded in fp64.  The group
# takes the lowest t of smallest E_t (strictly smaller replaces), and its
# codes are that type's.  Packing appends, after the scale blocks, 8 bytes per
# unit t = strip * G + g: byte rq (0..7) holds the types of rows rq + 8 i,
# i = 0..3, in bits 2i + 1 : 2i.

MAX_TYPES = {4: 4, 3: 2}
TYPE_BLOCK = 8       # bytes of one unit's group types


def _normalised(w) -> Tuple[np.ndarray, np.ndarray]:
    """Per group of 128: v = fp32(w) / fp32(s) with s the absolute maximum
    (v = 0 when s == 0), as quantize() computes them; (v[N, G, 128], s[N, G])."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    wg = w.reshape(n, k // GROUP, GROUP)
    s = np.max(np.abs(wg), axis=2)
    s_b = np.broadcast_to(s[:, :, None], wg.shape)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s_b > 0, wg / s_b, np.float32(0.0)).astype(np.float32)
    return v, s


def type_errors(w, type_levels, bits: int) -> np.ndarray:
    """E[t, n, g] (fp64): each type's squared RTN error over the group, summed
    over k in increasing order."""
    levels = [np.asarray(l, dtype=np.float32) for l in type_levels]
    v, _ = _normalised(w)
    n, g, _ = v.shape
    errs = np.zeros((len(levels), n, g), dtype=np.float64)
    for t, lv in enumerate(levels):
        codes, _ = quantize(w, lv, bits)
        c = lv[codes.reshape(n, g, GROUP)]                   # float32 levels
        d = (v - c).astype(np.float32).astype(np.float64)    # the fp32 difference
        for kk in range(GROUP):                              # k = 0, 1, ..., 127
            errs[t] = errs[t] + d[:, :, kk] * d[:, :, kk]
    return errs


def quantize_typed(w, type_levels, bits: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(codes uint8[N, K], scale bits uint16[N, G], types uint8[N, G]): every
    group quantized with the type of smallest error (lowest index on ties)."""
    if bits not in MAX_TYPES:
        raise ValueError("bits must be 3 or 4")
    if not 1 <= len(type_levels) <= MAX_TYPES[bits]:
        raise ValueError("number of types")
    errs = type_errors(w, type_levels, bits)
    n, g = errs.shape[1:]
    best = np.zeros((n, g), dtype=np.uint8)
    best_e = errs[0].copy()
    for t in range(1, len(type_levels)):
        take = errs[t] < best_e
        best[take] = t
        best_e[take] = errs[t][take]
    codes = np.zeros((n, g * GROUP), dtype=np.uint8)
    sb = None
    for t, lv in enumerate(type_levels):
        q_t, sb = quantize(w, lv, bits)
        pick = np.repeat(best == t, GROUP, axis=1)
        codes[pick] = q_t[pick]
    return codes, sb, best


def packed_bytes_typed(n: int, k: int, bits: int) -> int:
    return packed_bytes(n, k, bits) + (n // STRIP) * (k // GROUP) * TYPE_BLOCK


def pack_typed(codes, scale_bits, types, bits: int) -> np.ndarray:
    """pack() followed by the type blocks (8 bytes per unit)."""
    q = np.asarray(codes, dtype=np.uint8)
    n, k = q.shape
    ty = np.asarray(types, dtype=np.uint8)
    g = k // GROUP
    if ty.shape != (n, g):
        raise ValueError("types shape mismatch")
    if np.any(ty >= MAX_TYPES[bits]):
        raise ValueError("type out of range")
    body = pack(q, scale_bits, bits)
    # row r = 8 i + rq of strip s -> bits 2i+1:2i of byte rq of unit (s, g)
    t4 = ty.reshape(n // STRIP, 4, 8, g).astype(np.uint32)      # [s, i, rq, g]
    byte = np.zeros((n // STRIP, 8, g), dtype=np.uint32)
    for i in range(4):
        byte |= t4[:, i] << (2 * i)
    blocks = byte.transpose(0, 2, 1).astype(np.uint8)             # [s, g, rq]
    return np.concatenate([body, np.ascontiguousarray(blocks).reshape(-1)])


def unpack_typed(packed, n: int, k: int, bits: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Inverse of pack_typed, the type bytes read one by one."""
    p = np.asarray(packed, dtype=np.uint8)
    if p.size != packed_bytes_typed(n, k, bits):
        raise ValueError("packed size mismatch")
    body = packed_bytes(n, k, bits)
    q, sb = unpack(p[:body], n, k, bits)
    g = k // GROUP
    ty = np.zeros((n, g), dtype=np.uint8)
    for row in range(n):
        s, r = divmod(row, STRIP)
        for gi in range(g):
            byte = int(p[body + (s * g + gi) * TYPE_BLOCK + r % 8])
            ty[row, gi] = (byte >> (2 * (r // 8))) & 3
    return q, sb, ty


def typed_levels(types, type_levels) -> np.ndarray:
    """c[n, g, i]: the levels (fp64) of each group's type."""
    table = np.stack([np.asarray(l, dtype=np.float64) for l in type_levels])
    return table[np.asarray(types)]


def dequant_typed(codes, scale_bits, types, type_levels) -> np.ndarray:
    """W_hat[n, k] = s[n, g] * c_{type[n, g]}[q[n, k]] in fp64 (exact)."""
    q = np.asarray(codes)
    n, k = q.shape
    c = typed_levels(types, type_levels)                          # [N, G, L]
    qg = q.reshape(n, k // GROUP, GROUP)
    vals = np.take_along_axis(c, qg.astype(np.int64), axis=2)     # [N, G, 128]
    s = bf16_bits_to_f32(scale_bits).astype(np.float64)
    return (vals * s[:, :, None]).reshape(n, k)


def gemv_typed(x, codes, scale_bits, types, type_levels) -> np.ndarray:
    """y[m, n] = sum_g s[n, g] * sum_{k in g} x[m, k] * c_{type[n, g]}[q[n, k]]
    in fp64: the per-group partial sum with the group's own levels, rescaled
    once per group."""
    xf = np.asarray(x, dtype=np.float64)
    q = np.asarray(codes)
    n, k = q.shape
    m = xf.shape[0]
    g = k // GROUP
    c = typed_levels(types, type_levels)
    cq = np.take_along_axis(c, q.reshape(n, g, GROUP).astype(np.int64), axis=2)  # [N, G, 128]
    xg = xf.reshape(m, g, GROUP)
    partial = np.einsum("mgk,ngk->gmn", xg, cq)                   # [G, M, N]
    s = bf16_bits_to_f32(scale_bits).astype(np.float64)
    return np.sum(partial * s.T[:, None, :], axis=0)


def gemv_rows(x, w_rows, levels_f32, bits: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Quantize a subset of rows and return (codes, scale bits, y[:, rows]).

    Rows are independent in both quantization and the product, so checking a
    sample of rows of a large layer needs only those rows."""
    codes, sb = quantize(w_rows, levels_f32, bits)
    return codes, sb, gemv(x, codes, sb, levels_f32)


def rel_error_gate(y, y_ref, floor_frac: float = 1e-2) -> float:
    """max |y - y_ref| / max(|y_ref|, floor_frac * rms of y_ref's row), the
    error measure the 2e-3 tolerance applies to.  The floor keeps outputs
    that cancel to near zero from dominating a relative measure."""
    y = np.asarray(y, dtype=np.float64)
    r = np.asarray(y_ref, dtype=np.float64)
    rms = np.sqrt(np.mean(np.square(r), axis=-1, keepdims=True))
    den = np.maximum(np.abs(r), floor_frac * rms)
    den = np.where(den > 0, den, 1.0)
    return float(np.max(np.abs(y - r) / den)) if r.size else 0.0
