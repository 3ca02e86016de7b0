"""Pins of the CPU oracle to things other than itself (CPU only).

Each test checks one oracle function against a closed form, an invariant, a
brute-force computation written differently, a library routine in a special
case, a literature table, or bytes derived by hand from the layout definition.
Chosen so that a plausible slip (a dropped term, a wrong sign, a swapped index,
a transposed operand, a flipped tie rule) fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.integrate
import torch

import workloads
from oracle import lutq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch_cast_on_fp32_values():
    # Library special case: for fp32 inputs a single round-to-nearest-even to
    # bf16 is exactly torch's fp32 -> bf16 cast.
    rng = np.random.default_rng(0)
    v = rng.standard_normal(200000).astype(np.float32) * np.float32(3.0)
    # add exact ties: bf16 grid points plus half an ulp
    grid = (rng.integers(0, 2**15, 5000).astype(np.uint32) << 16).view(np.float32)
    grid = grid[np.isfinite(grid) & (np.abs(grid) > 1e-30) & (np.abs(grid) < 1e30)]
    half_ulp = (grid.view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    v = np.concatenate([v, half_ulp])
    ours = O.bf16_round(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, ref)


def _rne_8bit_fraction(x: Fraction) -> Fraction:
    """Exact rational round-to-nearest-even to 8 significant bits."""
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = 0
    while x >= 2:
        x /= 2
        e += 1
    while x < 1:
        x *= 2
        e -= 1
    scaled = x * 128                       # in [128, 256)
    fl = scaled.numerator // scaled.denominator
    rem = scaled - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * Fraction(fl, 128) * (Fraction(2) ** e)


# ---------------------------------------------------------------- codebooks

def test_logb_codebook_closed_form_exact_rationals():
    # Log_bQuant abstract (logarithmic codebook, adjustable base); base 1.6 =
    # 8/5 so the levels are +-(5/8)^k exactly.  Rounded here with exact
    # rational arithmetic, independently of the oracle's float path.
    _, vals = O.codebook("logb", 4)
    expect_pos = [_rne_8bit_fraction(Fraction(5, 8) ** k) for k in range(8)]
    expect = sorted([-v for v in expect_pos] + expect_pos)
    assert [Fraction(float(v)) for v in vals] == expect
    # k <= 3 are exact dyadic rationals; k = 4 rounds by hand:
    # (5/8)^4 = 0.152587890625 = 1.220703125 * 2^-3; 1.2207.. * 128 = 156.25 -> 156
    assert list(vals[8:13]) == [float(_rne_8bit_fraction(Fraction(5, 8) ** 7)),
                                float(_rne_8bit_fraction(Fraction(5, 8) ** 6)),
                                float(_rne_8bit_fraction(Fraction(5, 8) ** 5)),
                                0.15234375, 0.244140625]
    assert list(vals[12:]) == [0.244140625, 0.390625, 0.625, 1.0]
    assert 0.0 not in vals
    assert np.all(np.diff(vals) > 0)
    np.testing.assert_array_equal(vals, -vals[::-1])


def _phi_cdf(z: float) -> float:
    return 0.5 * math.erfc(-z / math.sqrt(2.0))


def _phi_inv_bisect(p: float) -> float:
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if _phi_cdf(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_nf4_levels_are_normal_quantiles():
    # FLUTE abstract: NormalFloat lookup table.  The normal CDF here is
    # math.erfc, not the oracle's scipy quantile routine.
    lv = O.nf4_levels()
    assert lv.shape == (16,)
    assert np.all(np.diff(lv) > 0)
    assert lv[0] == -1.0 and lv[15] == 1.0 and lv[7] == 0.0
    assert np.sum(lv > 0) == 8 and np.sum(lv < 0) == 7
    delta = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))
    zmax = _phi_inv_bisect(delta)
    p_pos = [_phi_cdf(v * zmax) for v in lv[8:]]
    p_neg = [_phi_cdf(-v * zmax) for v in lv[:7]]
    np.testing.assert_allclose(sorted(p_pos), np.linspace(delta, 0.5, 9)[:-1][::-1],
                               rtol=0, atol=1e-12)
    np.testing.assert_allclose(sorted(p_neg), np.linspace(delta, 0.5, 8)[:-1][::-1],
                               rtol=0, atol=1e-12)


def test_nf4_bf16_rounding_not_near_a_tie():
    # Every level is far enough from a bf16 rounding boundary that a 1e-12
    # error in the quantile cannot change its bf16 value.
    lv = O.nf4_levels()
    for v in lv:
        if v == 0:
            continue
        m, e = math.frexp(abs(v))
        frac = (m * 256.0) % 1.0
        assert abs(frac - 0.5) > 1e-6


def _golden_lloyd():
    rows = {}
    with open(os.path.join(GOLDEN, "lloyd_max_gaussian_8.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            kind, idx, val = line.split()
            rows[(kind, int(idx))] = float(val)
    return rows


def test_lloyd_max_matches_max_1960_table():
    y, t = O.lloyd_max_normal(8)
    g = _golden_lloyd()
    for i in range(1, 5):
        assert abs(y[3 + i] - g[("output", i)]) < 6e-4
    for i in range(1, 4):
        assert abs(t[3 + i] - g[("threshold", i)]) < 6e-4
    assert abs(t[3]) < 1e-12
    # mean squared error of the quantizer, by numerical integration
    edges = [-np.inf] + list(t) + [np.inf]
    pdf = lambda z: math.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)
    mse = sum(scipy.integrate.quad(lambda z, c=y[i]: (z - c) ** 2 * pdf(z),
                                   edges[i], edges[i + 1])[0] for i in range(8))
    assert abs(mse - g[("mse", 0)]) < 2e-5


def test_lloyd_max_fixed_point_by_quadrature():
    # Each level is the centroid of its cell (computed by quadrature rather
    # than the closed form the oracle iterates) and each threshold the midpoint.
    y, t = O.lloyd_max_normal(8)
    edges = [-np.inf] + list(t) + [np.inf]
    pdf = lambda z: math.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)
    for i in range(8):
        mass = scipy.integrate.quad(pdf, edges[i], edges[i + 1], epsabs=1e-14)[0]
        mom = scipy.integrate.quad(lambda z: z * pdf(z), edges[i], edges[i + 1],
                                   epsabs=1e-14)[0]
        assert abs(mom / mass - y[i]) < 1e-9
    np.testing.assert_allclose(t, 0.5 * (y[:-1] + y[1:]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(y, -y[::-1], rtol=0, atol=1e-12)


def test_lloyd_max3_bf16_values():
    # normalised by the outermost level; hand-rounded to 8 significant bits:
    # 0.245094/2.151946 = 0.113894 -> 233/128 * 2^-4 = 0.11376953125, etc.
    _, vals = O.codebook("lloyd_max3", 3)
    assert list(vals[4:]) == [0.11376953125, 0.3515625, 0.625, 1.0]
    np.testing.assert_array_equal(vals, -vals[::-1])


def test_uniform4_levels():
    _, vals = O.codebook("uniform4", 4)
    assert vals[0] == -1.0 and vals[15] == 1.0
    np.testing.assert_array_equal(vals, -vals[::-1])


# ---------------------------------------------------------------- quantization

def _levels(kind, bits):
    return O.codebook(kind, bits)[1]


def _random_w(n, k, seed, scale=0.02):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((n, k), generator=g) * scale).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("logb", 4), ("lloyd_max3", 3),
                                       ("uniform4", 4)])
def test_quantize_matches_fp64_bruteforce_except_near_ties(kind, bits):
    # Group-128 RTN study: round to nearest.  Independent fp64 argmin over
    # every level, element by element.
    lv = _levels(kind, bits)
    w = _random_w(16, 256, seed=3)
    codes, sb = O.quantize(w, lv, bits)
    s = O.bf16_bits_to_f32(sb).astype(np.float64)
    mism = 0
    for n in range(16):
        for k in range(256):
            sc = s[n, k // 128]
            v = w[n, k] / sc if sc > 0 else 0.0
            d = [abs(v - float(c)) for c in lv]
            order = sorted(range(len(d)), key=lambda i: (d[i], i))
            if order[0] != codes[n, k]:
                assert d[order[1]] - d[order[0]] < 1e-6
                mism += 1
    assert mism <= 2


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("logb", 4), ("lloyd_max3", 3)])
def test_quantize_fp32_rule_by_stable_sort(kind, bits):
    # The same fp32 rule written a second way: a stable sort of the fp32
    # distances puts the lowest index of the minimum first.
    lv = _levels(kind, bits).astype(np.float32)
    w = _random_w(32, 512, seed=4)
    codes, sb = O.quantize(w, lv, bits)
    s = O.bf16_bits_to_f32(sb)
    v = (w.reshape(32, 4, 128) / s[:, :, None]).astype(np.float32).reshape(32, 512)
    d = np.abs(v[:, :, None] - lv[None, None, :]).astype(np.float32)
    first = np.argsort(d, axis=2, kind="stable")[:, :, 0]
    np.testing.assert_array_equal(codes, first)


def test_quantize_scale_is_group_absmax_and_argmax_maps_to_unit_level():
    lv = _levels("nf4", 4)
    w = _random_w(8, 384, seed=5)
    codes, sb = O.quantize(w, lv, 4)
    s = O.bf16_bits_to_f32(sb)
    wg = w.reshape(8, 3, 128)
    np.testing.assert_array_equal(s, np.abs(wg).max(axis=2))
    cg = codes.reshape(8, 3, 128)
    for n in range(8):
        for g in range(3):
            i = int(np.argmax(np.abs(wg[n, g])))
            assert lv[cg[n, g, i]] == np.sign(wg[n, g, i])
    # every dequantized value lies in {s * c_i} and |value| <= s
    wh = O.dequant(codes, sb, lv)
    for n in range(8):
        for g in range(3):
            allowed = set((s[n, g].astype(np.float64) * lv.astype(np.float64)).tolist())
            assert set(wh[n, g * 128:(g + 1) * 128].tolist()) <= allowed


def test_quantize_hand_example_nf4():
    # N = 1, K = 128: w_k = 0.5 * c_{k mod 16} (exact in bf16) -> s = 0.5 and
    # v = c_{k mod 16} exactly -> q_k = k mod 16.
    lv = _levels("nf4", 4)
    w = np.array([[0.5 * lv[k % 16] for k in range(128)]], dtype=np.float32)
    codes, sb = O.quantize(w, lv, 4)
    assert list(codes[0]) == [k % 16 for k in range(128)]
    assert O.bf16_bits_to_f32(sb)[0, 0] == 0.5


def test_quantize_zero_group_and_negative_zero():
    # All-zero group: v = 0.  NF4 has an exact 0 at index 7; the log table has
    # none and +-(5/8)^7 tie, so the lower index (the negative level) wins.
    z = np.zeros((1, 128), dtype=np.float32)
    z[0, 5] = -0.0
    c_nf4, s = O.quantize(z, _levels("nf4", 4), 4)
    assert np.all(c_nf4 == 7) and s[0, 0] == 0
    c_log, _ = O.quantize(z, _levels("logb", 4), 4)
    assert np.all(c_log == 7)
    c_lm, _ = O.quantize(z, _levels("lloyd_max3", 3), 3)
    assert np.all(c_lm == 3)


def test_quantize_subnormal_group_is_not_flushed():
    # Scaling a group by a power of two leaves every ratio w/s unchanged, so
    # the codes of a subnormal group equal those of the same group scaled up.
    # A flush-to-zero quantizer would give all-zero-group codes instead.
    # bf16 subnormals are m * 2^-133 with integer |m| < 128.
    lv = _levels("nf4", 4)
    m = np.random.default_rng(6).integers(-127, 128, size=(1, 128)).astype(np.float64)
    w = (m * 2.0 ** -10).astype(np.float32)
    tiny = (m * 2.0 ** -133).astype(np.float32)
    assert np.all(np.abs(tiny[tiny != 0]) < np.finfo(np.float32).tiny)
    assert np.array_equal(O.bf16_round(tiny.astype(np.float64)), tiny.astype(np.float64))
    c_big, _ = O.quantize(w, lv, 4)
    c_tiny, _ = O.quantize(tiny, lv, 4)
    np.testing.assert_array_equal(c_big, c_tiny)
    assert len(set(c_tiny[0].tolist())) > 4


def test_quantize_rejects_nonfinite():
    w = _random_w(1, 128, seed=7)
    w[0, 3] = np.inf
    with pytest.raises(ValueError):
        O.quantize(w, _levels("nf4", 4), 4)


# ---------------------------------------------------------------- packing

def _zero_scales(n, k):
    return np.zeros((n, k // 128), np.uint16)


def test_packed_size_formula():
    # codes (4 or 3 bits per weight) plus one 16-bit scale per 128 weights
    assert O.packed_bytes(4096, 14336, 4) == 4096 * 14336 // 2 + 4096 * 14336 // 64
    assert O.packed_bytes(4096, 4096, 3) == 3 * 4096 * 4096 // 8 + 4096 * 4096 // 64
    q = np.zeros((64, 256), np.uint8)
    assert O.pack(q, _zero_scales(64, 256), 4).size == 64 * 256 // 2 + 64 * 256 // 64
    assert O.pack(q, _zero_scales(64, 256), 3).size == 3 * 64 * 256 // 8 + 64 * 256 // 64


@pytest.mark.parametrize("bits", [3, 4])
def test_pack_unpack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    q = rng.integers(0, 1 << bits, size=(64, 384), dtype=np.uint8)
    sb = rng.integers(0, 1 << 16, size=(64, 3), dtype=np.uint16)
    q2, sb2 = O.unpack(O.pack(q, sb, bits), 64, 384, bits)
    np.testing.assert_array_equal(q2, q)
    np.testing.assert_array_equal(sb2, sb)


def test_pack_w4_hand_derived_bytes():
    n, k = 64, 256
    nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
    q = ((nn + kk + 5 * (kk // 32)) % 16).astype(np.uint8)
    p = O.pack(q, _zero_scales(n, k), 4)
    with open(os.path.join(GOLDEN, "pack_v2_w4_pattern.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            off = int(parts[0])
            want = bytes(int(b, 16) for b in parts[1:])
            assert bytes(p[off:off + 16]) == want, off


def test_pack_scales_hand_derived_bytes():
    n, k = 64, 256
    nn, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
    sb = (0x3C00 + 4 * nn + gg).astype(np.uint16)
    p = O.pack(np.zeros((n, k), np.uint8), sb, 4)
    seen = 0
    with open(os.path.join(GOLDEN, "pack_v2_scales.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            off = int(parts[0])
            assert bytes(p[off:off + 2]) == bytes(int(b, 16) for b in parts[1:]), off
            seen += 1
    assert seen == 5
    # every code byte is zero; the scale blocks hold all 128 scales once
    assert not p[:8192].any()
    assert sorted(p[8192:].copy().view("<u2").tolist()) == sorted(sb.reshape(-1).tolist())


def test_pack_w3_hand_derived_probes():
    with open(os.path.join(GOLDEN, "pack_v2_w3_probes.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            left, right = line.split("|")
            _, row, kk, qv = left.split()
            q = np.zeros((32, 128), np.uint8)
            q[int(row), int(kk)] = int(qv)
            p = O.pack(q, _zero_scales(32, 128), 3)
            vals = right.split()
            want = {int(vals[i]): int(vals[i + 1], 16) for i in range(0, len(vals), 2)}
            nz = {int(i): int(p[i]) for i in np.nonzero(p)[0]}
            assert nz == want, line


# ---------------------------------------------------------------- product

def test_gemv_equals_dequantize_then_matmul():
    # Library special case: numpy's fp64 matmul of x with the dequantized
    # matrix (scale applied per weight, not per group partial).
    lv = _levels("logb", 4)
    w = _random_w(64, 512, seed=8)
    codes, sb = O.quantize(w, lv, 4)
    g = torch.Generator().manual_seed(9)
    x = torch.randn((3, 512), generator=g).to(torch.bfloat16).float().numpy()
    y = O.gemv(x, codes, sb, lv)
    wh = O.dequant(codes, sb, lv)
    ref = x.astype(np.float64) @ wh.T
    bound = np.abs(x.astype(np.float64)) @ np.abs(wh).T
    assert np.all(np.abs(y - ref) <= 1e-13 * bound + 1e-300)


def test_gemv_exact_sum_bruteforce():
    # Pure-Python loops with math.fsum (exactly rounded sum) on a tiny case.
    lv = _levels("nf4", 4)
    w = _random_w(4, 256, seed=10)
    codes, sb = O.quantize(w, lv, 4)
    s = O.bf16_bits_to_f32(sb)
    g = torch.Generator().manual_seed(11)
    x = torch.randn((2, 256), generator=g).to(torch.bfloat16).float().numpy()
    y = O.gemv(x, codes, sb, lv)
    for m in range(2):
        for n in range(4):
            terms = [float(x[m, k]) * float(s[n, k // 128]) * float(lv[codes[n, k]])
                     for k in range(256)]
            exact = math.fsum(terms)
            assert abs(y[m, n] - exact) <= 1e-15 * math.fsum(abs(t) for t in terms)


def test_gemv_one_hot_is_the_dequantized_weight():
    lv = _levels("lloyd_max3", 3)
    w = _random_w(32, 256, seed=12)
    codes, sb = O.quantize(w, lv, 3)
    wh = O.dequant(codes, sb, lv)
    for k in (0, 1, 127, 128, 255):
        x = np.zeros((1, 256), np.float32)
        x[0, k] = 1.0
        np.testing.assert_array_equal(O.gemv(x, codes, sb, lv)[0], wh[:, k])


def test_gemv_hand_example():
    # w_k = 0.5 c_{k mod 16}, x_k = 1 if k mod 16 >= 8: each of c_8..c_15
    # appears 8 times, so y = 8 * 0.5 * sum_{i >= 8} c_i.
    lv = _levels("nf4", 4)
    w = np.array([[0.5 * lv[k % 16] for k in range(128)]], dtype=np.float32)
    codes, sb = O.quantize(w, lv, 4)
    x = np.array([[1.0 if k % 16 >= 8 else 0.0 for k in range(128)]], np.float32)
    y = O.gemv(x, codes, sb, lv)
    assert y[0, 0] == 4.0 * math.fsum(float(c) for c in lv[8:])


def test_gemv_linearity_and_row_permutation():
    lv = _levels("nf4", 4)
    w = _random_w(32, 256, seed=13)
    codes, sb = O.quantize(w, lv, 4)
    g = torch.Generator().manual_seed(14)
    x = torch.randn((2, 256), generator=g).to(torch.bfloat16).float().numpy()
    y = O.gemv(x, codes, sb, lv)
    np.testing.assert_array_equal(O.gemv(2 * x, codes, sb, lv), 2 * y)
    perm = np.random.default_rng(0).permutation(32)
    yp = O.gemv(x, codes[perm], sb[perm], lv)
    np.testing.assert_array_equal(yp, y[:, perm])


def test_rel_error_gate():
    r = np.array([[1.0, -2.0, 0.0, 4.0]])
    assert O.rel_error_gate(r, r) == 0.0
    y = r.copy()
    y[0, 3] += 4e-3
    assert abs(O.rel_error_gate(y, r) - 1e-3) < 1e-12
    y = r.copy()
    y[0, 2] = 1e-3          # floor = 1e-2 * rms(r) = 1e-2 * sqrt(21/4)
    assert abs(O.rel_error_gate(y, r) - 1e-3 / (1e-2 * math.sqrt(21 / 4))) < 1e-12


# ---------------------------------------------------------------- Hadamard rotation

def _parity_sign(i, j):
    return -1.0 if bin(i & j).count("1") % 2 else 1.0


def test_hadamard_closed_form_and_library():
    import scipy.linalg
    h = O.hadamard(128)
    want = np.array([[_parity_sign(i, j) for j in range(128)] for i in range(128)])
    np.testing.assert_array_equal(h, want)                          # (-1)^popcount(i & j)
    np.testing.assert_array_equal(h, scipy.linalg.hadamard(128))    # library construction
    np.testing.assert_array_equal(h @ h.T, 128.0 * np.eye(128))


def test_rht_of_unit_vectors_is_a_signed_hadamard_column():
    signs = workloads.rht_signs(5).numpy().astype(np.float64)
    w = np.zeros((3, 256))
    cases = [(0, 7, 1.0), (1, 228, 1.0), (2, 255, -2.0)]
    for row, k, val in cases:
        w[row, k] = val
    r = O.rht_weights(w, signs)
    x = O.rht_activations(w, signs)
    for row, k, val in cases:
        g, j = divmod(k, 128)
        col = np.array([_parity_sign(i, j) for i in range(128)]) * signs[j] * val
        np.testing.assert_array_equal(r[row, 128 * g:128 * g + 128], col)
        np.testing.assert_array_equal(x[row, 128 * g:128 * g + 128], col / 128.0)
        rest = np.delete(r[row], np.arange(128 * g, 128 * g + 128))
        assert not rest.any()


def test_rht_pair_preserves_inner_products_exactly():
    # small-integer data: every rotated weight is an integer in [-128, 128] and
    # every rotated activation that over 128, all exact in bf16
    rng = np.random.default_rng(3)
    w = rng.integers(-1, 2, size=(5, 384)).astype(np.float64)
    x = rng.integers(-1, 2, size=(2, 384)).astype(np.float64)
    signs = workloads.rht_signs(9).numpy()
    rw, rx = O.rht_weights(w, signs), O.rht_activations(x, signs)
    np.testing.assert_array_equal(rx @ rw.T, x @ w.T)


def test_rht_twice_with_plus_signs_scales_by_128():
    rng = np.random.default_rng(4)
    w = rng.integers(-1, 2, size=(4, 256)).astype(np.float64)
    ones = np.ones(128)
    np.testing.assert_array_equal(O.rht_weights(O.rht_weights(w, ones), ones), 128.0 * w)


def test_rht_rejects_bad_signs():
    w = np.zeros((1, 128))
    with pytest.raises(ValueError):
        O.rht_weights(w, np.zeros(128))
    with pytest.raises(ValueError):
        O.rht_activations(w, np.ones(64))


def test_rht_lowers_quantization_error_with_outliers():
    # the reason for the rotation: spreading a group's outliers over all 128
    # coordinates before round-to-nearest lowers the product's error
    w = workloads.normal_weights(64, 1024, 0.02, seed=12, outlier_frac=1e-2).float().numpy()
    x = workloads.activations(4, 1024, seed=13).float().numpy()
    signs = workloads.rht_signs(14).numpy()
    lv = _levels("nf4", 4)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    codes, sb = O.quantize(w, lv, 4)
    err_plain = np.linalg.norm(O.gemv(x, codes, sb, lv) - exact)
    wr = O.rht_weights(w, signs).astype(np.float32)
    xr = O.rht_activations(x, signs).astype(np.float32)
    codes_r, sb_r = O.quantize(wr, lv, 4)
    err_rht = np.linalg.norm(O.gemv(xr, codes_r, sb_r, lv) - exact)
    assert err_rht < 0.9 * err_plain


# ---------------------------------------------------------------- codebook fitted to a layer

def test_fit_histogram_hand_values():
    w = np.zeros((1, 256), np.float32)
    w[0, :4] = [2.0, -2.0, 1.0, -0.5]       # group 0: s = 2 -> v = 1, -1, 0.5, -0.25, then 124 zeros
    h = O.fit_histogram(w)                   # group 1 is all zero (s = 0): 128 zeros
    want = np.zeros(O.HIST_BINS, np.int64)
    want[O.HIST_BINS - 1] += 1               # v = 1: (1 + 1) * 8192 = 16384, clamped
    want[0] += 1                             # v = -1
    want[12288] += 1                         # v = 0.5: 1.5 * 8192
    want[6144] += 1                          # v = -0.25: 0.75 * 8192
    want[8192] += 124 + 128                  # v = 0
    np.testing.assert_array_equal(h, want)


def test_fit_two_clusters_lands_on_their_centres():
    h = np.zeros(O.HIST_BINS, np.int64)
    h[1000] = 10
    h[15000] = 30
    got = O.fit_codebook(h, np.array([-0.5, 0.5]))
    centres = (2 * np.array([1000, 15000]) + 1 - O.HIST_BINS) / O.HIST_BINS
    np.testing.assert_array_equal(got, O.bf16_round(centres))
    # a level whose cell stays empty keeps its starting value
    got3 = O.fit_codebook(h, np.array([-0.5, 0.25, 0.5]))
    assert got3[0] == O.bf16_round(np.array([centres[0]]))[0] and got3[1] == 0.25


def _hist_distortion(h, levels):
    c = (2 * np.arange(O.HIST_BINS) + 1 - O.HIST_BINS) / O.HIST_BINS
    d = np.min(np.abs(c[:, None] - np.asarray(levels)[None, :]), axis=1)
    return float(np.sum(h * d * d))


def test_fit_lowers_the_layers_distortion():
    w = workloads.student_t_weights(256, 1024, 5, 0.02, seed=21, outlier_frac=1e-3).float().numpy()
    h = O.fit_histogram(w)
    assert h.sum() == w.size
    for kind, bits in (("nf4", 4), ("lloyd_max3", 3)):
        _, init = O.codebook(kind, bits)
        fitted = O.fit_codebook(h, init)
        assert np.all(np.diff(fitted) > 0)
        assert _hist_distortion(h, fitted) < 0.97 * _hist_distortion(h, init)
