"""Property checks of the oracle on small random inputs (CPU): packing is a
bijection for any codes, scales and types; RTN picks a nearest level; every
typed choice is a type of smallest error; the products are linear in x."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import lutq_oracle as O

SETTINGS = settings(max_examples=25, deadline=None)


@SETTINGS
@given(st.integers(1, 3), st.integers(1, 3), st.sampled_from([3, 4]), st.integers(0, 2**31 - 1))
def test_pack_typed_is_a_bijection(strips, groups, bits, seed):
    rng = np.random.default_rng(seed)
    n, k = 32 * strips, 128 * groups
    codes = rng.integers(0, 1 << bits, size=(n, k), dtype=np.uint8)
    sb = rng.integers(0, 0x7f80, size=(n, groups)).astype(np.uint16)
    ty = rng.integers(0, O.MAX_TYPES[bits], size=(n, groups)).astype(np.uint8)
    p = O.pack_typed(codes, sb, ty, bits)
    assert p.size == O.packed_bytes_typed(n, k, bits)
    c2, s2, t2 = O.unpack_typed(p, n, k, bits)
    assert np.array_equal(c2, codes) and np.array_equal(s2, sb) and np.array_equal(t2, ty)


@SETTINGS
@given(st.sampled_from(["nf4", "logb", "uniform4"]), st.integers(0, 2**31 - 1))
def test_rtn_code_is_a_nearest_level(kind, seed):
    rng = np.random.default_rng(seed)
    w = O.bf16_round(rng.standard_normal((2, 256)) * 0.02).astype(np.float32)
    _, lv = O.codebook(kind, 4)
    codes, sb = O.quantize(w, lv, 4)
    s = np.repeat(O.bf16_bits_to_f32(sb), 128, axis=1)
    v = (w / s).astype(np.float32)
    d = np.abs(v[..., None] - lv).astype(np.float32)       # fp32 distances to every level
    assert np.all(d[np.arange(2)[:, None], np.arange(256)[None], codes] == d.min(axis=-1))


@SETTINGS
@given(st.integers(1, 4), st.integers(0, 2**31 - 1))
def test_typed_choice_has_the_smallest_error(t, seed):
    rng = np.random.default_rng(seed)
    w = O.bf16_round(rng.standard_t(4, size=(32, 256)) * 0.02).astype(np.float32)
    kinds = ["nf4", "logb", "uniform4", "nf4"][:t]
    tables = [O.codebook(k_, 4)[1] for k_ in kinds]
    errs = O.type_errors(w, tables, 4)
    _, _, ty = O.quantize_typed(w, tables, 4)
    chosen = np.take_along_axis(errs, ty[None].astype(np.int64), axis=0)[0]
    assert np.all(chosen == errs.min(axis=0))
    # and the lowest such type
    first = np.argmax(errs == errs.min(axis=0)[None], axis=0)
    assert np.array_equal(ty, first.astype(np.uint8))


@SETTINGS
@given(st.integers(0, 2**31 - 1))
def test_typed_product_is_linear_in_x(seed):
    rng = np.random.default_rng(seed)
    w = O.bf16_round(rng.standard_normal((32, 256)) * 0.02).astype(np.float32)
    tables = [O.codebook(k_, 4)[1] for k_ in ("nf4", "uniform4")]
    codes, sb, ty = O.quantize_typed(w, tables, 4)
    x1 = O.bf16_round(rng.standard_normal((1, 256))).astype(np.float32)
    x2 = O.bf16_round(rng.standard_normal((1, 256))).astype(np.float32)
    y1 = O.gemv_typed(x1, codes, sb, ty, tables)
    y2 = O.gemv_typed(x2, codes, sb, ty, tables)
    y12 = O.gemv_typed(x1 + x2, codes, sb, ty, tables)
    assert np.allclose(y12, y1 + y2, rtol=1e-12, atol=1e-12)
    assert np.array_equal(O.gemv_typed(2 * x1, codes, sb, ty, tables), 2 * y1)
