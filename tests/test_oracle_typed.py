"""Pins of the oracle's per-group data types (BitMoD abstract, "Daily Papers"
listing: each group of 128 weights may be quantized with its own numerical
data type), CPU only.  The selection is checked against exact rational
errors, special cases that reduce to plain RTN, groups built from one type's
levels, the tie rule, an invariant (more types never raise a group's error)
and bytes derived by hand from the layout definition."""
import os
from fractions import Fraction

import numpy as np
import pytest

import workloads
from oracle import lutq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
KINDS4 = ("nf4", "logb", "uniform4")


def _levels(kind, bits=4):
    return O.codebook(kind, bits)[1]


def _weights(n, k, seed, outlier_frac=1e-2):
    return workloads.normal_weights(n, k, 0.02, seed=seed, outlier_frac=outlier_frac).float().numpy()


@pytest.mark.parametrize("bits,kind", [(4, "nf4"), (4, "logb"), (3, "lloyd_max3")])
def test_single_type_is_plain_rtn(bits, kind):
    w = _weights(64, 384, seed=1)
    lv = _levels(kind, bits)
    codes, sb, ty = O.quantize_typed(w, [lv], bits)
    c0, sb0 = O.quantize(w, lv, bits)
    np.testing.assert_array_equal(codes, c0)
    np.testing.assert_array_equal(sb, sb0)
    assert not ty.any()


def test_groups_built_from_one_type_select_it():
    # each group is 0.5 * (levels of one type), both ends (-1, +1) included so
    # that s = 0.5 and v is the level itself: that type's error is exactly 0
    rng = np.random.default_rng(5)
    tables = [_levels(k) for k in KINDS4]
    n, g = 32, 6
    want = rng.integers(0, 3, size=(n, g))
    w = np.zeros((n, g, 128), np.float32)
    for r in range(n):
        for gi in range(g):
            lv = tables[want[r, gi]]
            idx = rng.integers(0, 16, size=128)
            idx[0], idx[1] = 0, 15
            w[r, gi] = 0.5 * lv[idx]
    w = w.reshape(n, g * 128)
    errs = O.type_errors(w, tables, 4)
    codes, sb, ty = O.quantize_typed(w, tables, 4)
    np.testing.assert_array_equal(ty, want)
    assert np.all(np.take_along_axis(errs, want[None], axis=0) == 0.0)
    np.testing.assert_array_equal(O.dequant_typed(codes, sb, ty, tables), w)


def _exact_errors(w, tables, bits):
    """E[t, n, g] with exact rational differences v - c (no fp32 rounding of
    the difference, no rounding of the sum)."""
    n, k = w.shape
    wg = w.reshape(n, k // 128, 128)
    out = np.zeros((len(tables), n, k // 128), dtype=object)
    for t, lv in enumerate(tables):
        codes, _ = O.quantize(w, lv, bits)
        cg = codes.reshape(n, k // 128, 128)
        for r in range(n):
            for gi in range(k // 128):
                s = np.float32(np.max(np.abs(wg[r, gi])))
                tot = Fraction(0)
                for kk in range(128):
                    v = np.float32(wg[r, gi, kk]) / s if s > 0 else np.float32(0.0)
                    d = Fraction(float(v)) - Fraction(float(lv[cg[r, gi, kk]]))
                    tot += d * d
                out[t, r, gi] = tot
    return out


@pytest.mark.parametrize("bits,kinds", [(4, KINDS4), (3, ("lloyd_max3", None))])
def test_choice_is_the_exact_argmin_except_near_ties(bits, kinds):
    if bits == 3:
        lm = _levels("lloyd_max3", 3)
        tables = [lm, O.bf16_round(lm * np.float32(0.9)).astype(np.float32)]
        tables[1][0], tables[1][-1] = -1.0, 1.0    # a second 3-bit type: shrunk interior
    else:
        tables = [_levels(k) for k in kinds]
    w = _weights(12, 512, seed=7)
    _, _, ty = O.quantize_typed(w, tables, bits)
    exact = _exact_errors(w, tables, bits)
    # every error itself: within the fp32 rounding of the 128 differences
    errs = O.type_errors(w, tables, bits)
    ex = exact.astype(np.float64)
    assert np.all(np.abs(errs - ex) <= 1e-6 * ex + 1e-30)
    near = 0
    for r in range(w.shape[0]):
        for gi in range(w.shape[1] // 128):
            e = [exact[t, r, gi] for t in range(len(tables))]
            best = min(e)
            chosen = e[int(ty[r, gi])]
            if chosen != best:
                # the fp32 differences may only flip a choice between errors
                # within a relative 1e-6 of each other
                assert float((chosen - best) / best) < 1e-6
                near += 1
    assert near <= 1
    # the choice is not constant on this data (the pin can fail)
    assert len(np.unique(ty)) > 1


def test_ties_take_the_lowest_type():
    w = _weights(32, 256, seed=9)
    nf4 = _levels("nf4")
    _, _, ty = O.quantize_typed(w, [nf4, nf4.copy()], 4)
    assert not ty.any()
    uni = _levels("uniform4")
    _, _, ty2 = O.quantize_typed(w, [uni, nf4, uni.copy()], 4)
    assert not np.any(ty2 == 2)
    assert np.any(ty2 == 0) or np.any(ty2 == 1)


def test_more_types_never_raise_a_groups_error():
    w = _weights(64, 512, seed=11)
    tables = [_levels(k) for k in KINDS4]
    errs = O.type_errors(w, tables, 4)
    prev = None
    for t in range(1, 4):
        _, _, ty = O.quantize_typed(w, tables[:t], 4)
        e = np.take_along_axis(errs[:t], ty[None].astype(np.int64), axis=0)[0]
        assert np.all(e == errs[:t].min(axis=0))
        if prev is not None:
            assert np.all(e <= prev)
        prev = e


def test_type_count_limits():
    w = _weights(32, 128, seed=2)
    lv4 = _levels("nf4")
    with pytest.raises(ValueError):
        O.quantize_typed(w, [lv4] * 5, 4)
    lv3 = _levels("lloyd_max3", 3)
    with pytest.raises(ValueError):
        O.quantize_typed(w, [lv3] * 3, 3)
    with pytest.raises(ValueError):
        O.quantize_typed(w, [], 4)


def test_pack_typed_hand_derived_bytes():
    n, k = 64, 256
    nn, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
    ty = (((nn % 8) + (nn // 8) + gg) % 4).astype(np.uint8)
    p = O.pack_typed(np.zeros((n, k), np.uint8), np.zeros((n, 2), np.uint16), ty, 4)
    assert p.size == O.packed_bytes_typed(n, k, 4) == 8448 + 32
    seen = 0
    with open(os.path.join(GOLDEN, "pack_v2_types.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            off, byte = line.split()
            assert int(p[int(off)]) == int(byte, 16), off
            seen += 1
    assert seen == 5
    assert not p[:8448].any()


@pytest.mark.parametrize("bits", [3, 4])
def test_pack_typed_roundtrip_and_body(bits):
    rng = np.random.default_rng(bits)
    n, k = 96, 384
    codes = rng.integers(0, 1 << bits, size=(n, k), dtype=np.uint8)
    sb = rng.integers(0, 0x7f80, size=(n, k // 128)).astype(np.uint16)
    ty = rng.integers(0, O.MAX_TYPES[bits], size=(n, k // 128)).astype(np.uint8)
    p = O.pack_typed(codes, sb, ty, bits)
    body = O.packed_bytes(n, k, bits)
    np.testing.assert_array_equal(p[:body], O.pack(codes, sb, bits))
    c2, s2, t2 = O.unpack_typed(p, n, k, bits)
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(s2, sb)
    np.testing.assert_array_equal(t2, ty)
    bad = ty.copy()
    bad[3, 1] = O.MAX_TYPES[bits]
    with pytest.raises(ValueError):
        O.pack_typed(codes, sb, bad, bits)


def test_dequant_typed_hand_example():
    # one row, two groups: group 0 with type 0 (uniform4), group 1 with type
    # 1 (logb); codes k % 16; scales 0.5 and 0.25
    uni, logb = _levels("uniform4"), _levels("logb")
    codes = (np.arange(256) % 16).astype(np.uint8)[None]
    sb = O.bf16_bits(np.array([[0.5, 0.25]]))
    ty = np.array([[0, 1]], np.uint8)
    wh = O.dequant_typed(codes, sb, ty, [uni, logb])
    # uniform4 level 3 = (2*3 - 15) / 15 = -0.6 -> bf16; logb level 15 = 1
    assert wh[0, 3] == 0.5 * float(O.bf16_round(np.array([-0.6]))[0])
    assert wh[0, 128 + 15] == 0.25
    # logb level 8 = +1.6^-7 (the smallest positive magnitude) -> bf16
    assert wh[0, 128 + 8] == 0.25 * float(O.bf16_round(np.array([1.6 ** -7]))[0])


def test_gemv_typed_exact_sum_and_one_hot():
    rng = np.random.default_rng(3)
    tables = [_levels(k) for k in KINDS4]
    w = _weights(32, 256, seed=4)
    codes, sb, ty = O.quantize_typed(w, tables, 4)
    x = O.bf16_round(rng.standard_normal((2, 256))).astype(np.float32)
    y = O.gemv_typed(x, codes, sb, ty, tables)
    # brute force with exact rationals on a few outputs
    s = O.bf16_bits_to_f32(sb)
    for m, nrow in ((0, 0), (1, 17), (0, 31)):
        tot = Fraction(0)
        for kk in range(256):
            c = tables[ty[nrow, kk // 128]][codes[nrow, kk]]
            tot += Fraction(float(x[m, kk])) * Fraction(float(s[nrow, kk // 128])) * Fraction(float(c))
        assert abs(y[m, nrow] - float(tot)) <= 1e-12 * max(1.0, abs(float(tot)))
    # one-hot activations give the dequantized weights exactly
    e = np.zeros((1, 256), np.float32)
    e[0, 200] = 1.0
    np.testing.assert_array_equal(O.gemv_typed(e, codes, sb, ty, tables)[0],
                                  O.dequant_typed(codes, sb, ty, tables)[:, 200])
    # all groups of one type: the untyped product with that type's levels
    for t in range(3):
        same = np.full_like(ty, t)
        np.testing.assert_allclose(O.gemv_typed(x, codes, sb, same, tables),
                                   O.gemv(x, codes, sb, tables[t]), rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- per-row scale
# (Tetra abstract, aiqbench news item: one scale per matrix row)

@pytest.mark.parametrize("bits,kind", [(4, "nf4"), (3, "lloyd_max3")])
def test_rowscale_single_group_is_plain_rtn(bits, kind):
    # K = 128: the row is one group, so the two rules coincide
    w = _weights(64, 128, seed=21)
    lv = _levels(kind, bits)
    np.testing.assert_array_equal(O.quantize_rowscale(w, lv, bits)[0], O.quantize(w, lv, bits)[0])
    np.testing.assert_array_equal(O.quantize_rowscale(w, lv, bits)[1], O.quantize(w, lv, bits)[1])


def test_rowscale_equals_group_rtn_when_every_group_holds_the_row_max():
    w = _weights(32, 512, seed=22)
    m = np.max(np.abs(w), axis=1)
    for g in range(4):
        w[:, 128 * g + 7] = m                       # every group reaches the row maximum
    lv = _levels("nf4")
    c1, s1 = O.quantize_rowscale(w, lv, 4)
    c0, s0 = O.quantize(w, lv, 4)
    np.testing.assert_array_equal(c1, c0)
    np.testing.assert_array_equal(s1, s0)


def test_rowscale_scale_is_the_row_max_and_codes_by_brute_force():
    w = _weights(16, 384, seed=23)
    lv = _levels("logb")
    codes, sb = O.quantize_rowscale(w, lv, 4)
    s = O.bf16_bits_to_f32(sb)
    assert np.all(s == np.max(np.abs(w), axis=1)[:, None])
    # brute force in fp64 on the exact quotient: agrees except at near-ties
    v = w.astype(np.float64) / np.max(np.abs(w), axis=1, keepdims=True).astype(np.float64)
    d = np.abs(v[..., None] - lv.astype(np.float64))
    ref = np.argmin(d, axis=-1)
    srt = np.sort(d, axis=-1)
    tie = (srt[..., 1] - srt[..., 0]) < 1e-6
    assert np.all((codes == ref) | tie)
    assert np.mean(tie) < 1e-3
    # the row maximum maps to a +-1 level
    arg = np.argmax(np.abs(w), axis=1)
    assert np.all(np.abs(lv[codes[np.arange(16), arg]]) == 1.0)


# ------------------------------------------- tensor-wise asymmetric linear
# (Log_bQuant abstract: the asymmetric linear, tensor-wise baseline)

def test_tensorscale_is_rowscale_of_the_flattened_matrix_and_the_global_max():
    w = _weights(32, 256, seed=31)
    lv = _levels("uniform4")
    codes, sb = O.quantize_tensorscale(w, lv, 4)
    s = O.bf16_bits_to_f32(sb)
    assert np.all(s == np.max(np.abs(w)))
    c1, _ = O.quantize_rowscale(w.reshape(1, -1), lv, 4)
    np.testing.assert_array_equal(codes, c1.reshape(32, 256))
    # a single-row matrix: tensor scale = row scale
    np.testing.assert_array_equal(O.quantize_tensorscale(w[:1], lv, 4)[0],
                                  O.quantize_rowscale(w[:1], lv, 4)[0])


def test_asym_linear_levels_closed_form():
    lv = O.asym_linear_levels(-0.5, 1.0, 4)
    # (w_min + i (w_max - w_min) / 15) / 1.0 = -0.5 + 0.1 i, each rounded to bf16
    want = O.bf16_round(np.array([-0.5 + 0.1 * i for i in range(16)]))
    np.testing.assert_array_equal(lv, want)
    assert lv[0] == -0.5 and lv[-1] == 1.0
    assert np.all(np.diff(lv) > 0)
    lv3 = O.asym_linear_levels(-2.0, 0.5, 3)            # S = 2: from -1 to 0.25
    assert lv3[0] == -1.0 and lv3[-1] == 0.25 and lv3.size == 8
    np.testing.assert_array_equal(O.asym_linear_levels(0.0, 0.0, 4), np.zeros(16))
    with pytest.raises(ValueError):
        O.asym_linear_levels(1.0, -1.0, 4)


def test_asym_linear_grid_points_quantize_exactly():
    # weights on the (bf16) grid times S quantize to themselves
    lv = O.asym_linear_levels(-0.25, 1.0, 4).astype(np.float32)
    rng = np.random.default_rng(33)
    idx = rng.integers(0, 16, size=(32, 256))
    idx[0, 0] = 15                                       # the maximum, +1 * S
    w = (lv[idx] * np.float32(0.5)).astype(np.float32)  # S = 0.5, exact
    codes, sb = O.quantize_tensorscale(w, lv, 4)
    np.testing.assert_array_equal(codes, idx)
    np.testing.assert_array_equal(O.dequant(codes, sb, lv), w)


# ------------------------------------------------------------ group of 256

def test_group256_scale_is_the_256_max_and_codes_by_brute_force():
    w = _weights(16, 768, seed=41)
    lv = _levels("nf4")
    codes, sb = O.quantize_group256(w, lv, 4)
    s = O.bf16_bits_to_f32(sb)
    m256 = np.max(np.abs(w.reshape(16, 3, 256)), axis=2)
    np.testing.assert_array_equal(s, np.repeat(m256, 2, axis=1))
    v = w.astype(np.float64) / np.repeat(m256, 256, axis=1).astype(np.float64)
    d = np.abs(v[..., None] - lv.astype(np.float64))
    ref = np.argmin(d, axis=-1)
    srt = np.sort(d, axis=-1)
    tie = (srt[..., 1] - srt[..., 0]) < 1e-6
    assert np.all((codes == ref) | tie)


def test_group256_equals_group128_when_both_halves_share_the_max():
    w = _weights(32, 512, seed=42)
    m = np.max(np.abs(w.reshape(32, 2, 256)), axis=2)
    for j in range(2):
        w[:, 256 * j + 5] = m[:, j]
        w[:, 256 * j + 133] = -m[:, j]            # both 128-halves reach the 256 maximum
    lv = _levels("logb")
    c2, s2 = O.quantize_group256(w, lv, 4)
    c1, s1 = O.quantize(w, lv, 4)
    np.testing.assert_array_equal(c2, c1)
    np.testing.assert_array_equal(s2, s1)
    with pytest.raises(ValueError):
        O.quantize_group256(w[:, :384], lv, 4)


# ------------------------------------------------------------- group of 64

def test_group64_scales_codes_and_product():
    w = _weights(32, 256, seed=51)
    lv = _levels("nf4")
    codes, sb = O.quantize_group64(w, lv, 4)
    s = O.bf16_bits_to_f32(sb)
    np.testing.assert_array_equal(s, np.max(np.abs(w.reshape(32, 4, 64)), axis=2))
    v = w.astype(np.float64) / np.repeat(s, 64, axis=1).astype(np.float64)
    d = np.abs(v[..., None] - lv.astype(np.float64))
    srt = np.sort(d, axis=-1)
    tie = (srt[..., 1] - srt[..., 0]) < 1e-6
    assert np.all((codes == np.argmin(d, axis=-1)) | tie)
    # the product: the library matmul of the dequantized matrix
    x = O.bf16_round(np.random.default_rng(52).standard_normal((2, 256))).astype(np.float32)
    wh = lv.astype(np.float64)[codes] * np.repeat(s, 64, axis=1)
    np.testing.assert_allclose(O.gemv_group64(x, codes, sb, lv), x.astype(np.float64) @ wh.T,
                               rtol=1e-12, atol=1e-12)
    # groups of 64 whose two halves share the 128 maximum give the 128 result
    w2 = w.copy()
    m = np.max(np.abs(w2.reshape(32, 2, 128)), axis=2)
    for g in range(2):
        w2[:, 128 * g + 3] = m[:, g]
        w2[:, 128 * g + 70] = m[:, g]
    c64, s64 = O.quantize_group64(w2, lv, 4)
    c128, s128 = O.quantize(w2, lv, 4)
    np.testing.assert_array_equal(c64, c128)
    np.testing.assert_array_equal(s64[:, ::2], s128)


def test_pack_group64_hand_derived_scale_bytes():
    n, k = 64, 256
    nn, hh = np.meshgrid(np.arange(n), np.arange(4), indexing="ij")
    sb = (0x3C00 + 8 * nn + hh).astype(np.uint16)
    p = O.pack_group64(np.zeros((n, k), np.uint8), sb, 4)
    assert p.size == 8192 + 4 * 128
    seen = 0
    with open(os.path.join(GOLDEN, "pack_v2_scales_group64.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            off = int(parts[0])
            assert bytes(p[off:off + 2]) == bytes(int(b, 16) for b in parts[1:]), off
            seen += 1
    assert seen == 5
    assert sorted(p[8192:].copy().view("<u2").tolist()) == sorted(sb.reshape(-1).tolist())
