"""The C ABI without a GPU: the library loads, exports every function that
include/lutq.h declares, its host-only functions behave, and argument errors
come back before anything touches the device."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from oracle import lutq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"\b(lutq_[a-z0-9_]+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lq():
    import dequant_gemv_group_b200 as m
    return m


def test_library_exports_every_declared_function(lq):
    declared = _header_functions()
    assert {"lutq_quantize", "lutq_pack", "lutq_gemv", "lutq_gemm"} <= declared
    for name in sorted(declared):
        assert hasattr(lq.lib, name), name


def test_layout_version_and_sizes(lq):
    assert lq.lutq_layout_version() == O.LAYOUT_VERSION == 2
    for n, k, bits in [(4096, 14336, 4), (4096, 4096, 3), (32, 128, 4), (28672, 8192, 3)]:
        assert lq.lutq_packed_bytes(n, k, bits) == O.packed_bytes(n, k, bits)
    assert lq.lutq_packed_bytes(33, 128, 4) == -1
    assert lq.lutq_packed_bytes(32, 100, 4) == -1
    assert lq.lutq_packed_bytes(32, 128, 5) == -1
    assert lq.lutq_workspace_bytes(1, 4096, 14336, 4) > 0
    assert lq.lutq_workspace_bytes(0, 4096, 14336, 4) == -1


def test_status_strings(lq):
    for code in range(11):
        assert lq.lutq_status_string(code).startswith(lq._binding.STATUS_NAMES[code])
    assert "unknown" in lq.lutq_status_string(99)


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("logb", 4), ("lloyd_max3", 3),
                                       ("uniform4", 4)])
def test_host_codebook_bit_exact_vs_oracle(lq, kind, bits):
    import torch
    ours = lq.lutq_codebook(kind, bits).view(torch.int16).numpy().view(np.uint16)
    ref, _ = O.codebook(kind, bits)
    np.testing.assert_array_equal(ours, ref)


def test_codebook_bits_mismatch(lq):
    with pytest.raises(lq.LutqError) as e:
        lq.lutq_codebook("nf4", 3)
    assert e.value.status == 3


# Argument errors are decided on the host before any CUDA call, so fake (never
# dereferenced) 16-byte-aligned addresses are enough here.
A = 1 << 20


@pytest.mark.parametrize("name", ["lutq_quantize", "lutq_quantize_rowscale",
                                  "lutq_quantize_tensorscale", "lutq_quantize_group256"])
def test_quantize_argument_errors(lq, name):
    f = getattr(lq.lib, name)
    assert f(None, 32, 128, A, 4, A, A, None, None) == 1          # null W
    assert f(A, 32, 128, A, 5, A, A, None, None) == 3             # bits
    assert f(A, 33, 128, A, 4, A, A, None, None) == 2             # N % 32
    assert f(A, 32, 130, A, 4, A, A, None, None) == 2             # K % 128
    assert f(A, 0, 128, A, 4, A, A, None, None) == 2              # empty
    assert f(A + 2, 32, 256, A, 4, A, A, None, None) == 4         # misaligned


def test_pack_argument_errors(lq):
    f = lq.lib.lutq_pack
    assert f(None, A, 32, 128, 4, A, None, None) == 1
    assert f(A, None, 32, 128, 4, A, None, None) == 1             # null scales
    assert f(A, A, 32, 128, 2, A, None, None) == 3
    assert f(A, A, 64, 64, 4, A, None, None) == 2
    assert f(A, A, 32, 128, 4, A + 8, None, None) == 4
    assert f(A, A + 2, 32, 128, 4, A, None, None) == 4            # misaligned scales


@pytest.mark.parametrize("name", ["lutq_gemv", "lutq_gemm", "lutq_gemv_group64",
                                  "lutq_gemm_group64"])
def test_product_argument_errors(lq, name):
    f = getattr(lq.lib, name)
    ws = lq.lutq_workspace_bytes(1, 64, 256, 4)
    ok = dict(x=A, m=1, p=A, c=A, bits=4, n=64, k=256, y=A, ws=A, wsb=ws)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["x"], a["m"], a["p"], a["c"], a["bits"], a["n"], a["k"], a["y"],
                 a["ws"], a["wsb"], None, None)

    assert call(x=None) == 1
    assert call(p=None) == 1
    assert call(c=A + 8) == 4
    assert call(bits=2) == 3
    assert call(n=48) == 2
    assert call(k=200) == 2
    assert call(m=0) == 2
    if name.startswith("lutq_gemv"):
        assert call(m=17) == 2
    assert call(y=A + 4) == 4
    if ws > 0:
        assert call(ws=None) == 9
        assert call(wsb=ws - 1) == 9


def test_rht_argument_errors(lq):
    for f in (lq.lib.lutq_rht_weights, lq.lib.lutq_rht_activations):
        assert f(None, 32, 128, A, A + 4096, None) == 1              # null input
        assert f(A, 32, 128, None, A + 4096, None) == 1              # null signs
        assert f(A, 0, 128, A, A + 4096, None) == 2                  # no rows
        assert f(A, 32, 200, A, A + 4096 * 4, None) == 2             # K % 128
        assert f(A + 2, 32, 128, A, A + 1 << 16, None) == 4          # misaligned
        assert f(A, 32, 128, A, A + 2048, None) == 1                 # in and out overlap


def test_gemv_rht_argument_errors(lq):
    f = lq.lib.lutq_gemv_rht
    ws = lq.lutq_workspace_bytes(1, 64, 256, 4)

    def call(**kw):
        a = dict(dict(x=A, m=1, p=A, c=A, s=A, bits=4, n=64, k=256, y=A, ws=A, wsb=None), **kw)
        if a["wsb"] is None:  # a workspace of the problem's own size
            a["wsb"] = max(ws, lq.lutq_workspace_bytes(a["m"], a["n"], a["k"], 4))
        return f(a["x"], a["m"], a["p"], a["c"], a["s"], a["bits"], a["n"], a["k"], a["y"],
                 a["ws"], a["wsb"], None, None)

    assert call(s=None) == 1
    assert call(s=A + 4) == 4
    assert call(m=5) == 2                  # beyond the CUDA-core kernel: rotate and use lutq_gemm
    assert call(m=1, k=128 * 700) == 2     # activations too long for its shared memory
    assert call(bits=5) == 3


def test_typed_sizes_and_limits(lq):
    assert lq.lutq_max_types(4) == O.MAX_TYPES[4] == 4
    assert lq.lutq_max_types(3) == O.MAX_TYPES[3] == 2
    assert lq.lutq_max_types(5) == -1
    for n, k, bits in [(4096, 14336, 4), (4096, 4096, 3), (32, 128, 4)]:
        assert lq.lutq_packed_bytes_typed(n, k, bits) == O.packed_bytes_typed(n, k, bits)
    assert lq.lutq_packed_bytes_typed(33, 128, 4) == -1


def test_typed_argument_errors(lq):
    q = lq.lib.lutq_quantize_typed
    assert q(A, 32, 128, A, 2, 4, A, A, None, None, None) == 1     # null types output
    assert q(A, 32, 128, A, 0, 4, A, A, A, None, None) == 1        # no type
    assert q(A, 32, 128, A, 5, 4, A, A, A, None, None) == 1        # 5 types of 4-bit codes
    assert q(A, 32, 128, A, 3, 3, A, A, A, None, None) == 1        # 3 types of 3-bit codes
    assert q(A, 32, 128, A, 2, 5, A, A, A, None, None) == 3        # bits
    assert q(A, 33, 128, A, 2, 4, A, A, A, None, None) == 2        # N % 32
    assert q(A, 32, 128, A, 2, 4, A, A, A + 4, None, None) == 4    # misaligned types
    p = lq.lib.lutq_pack_typed
    assert p(A, A, None, 32, 128, 4, A, None, None) == 1
    assert p(A, A, A + 2, 32, 128, 4, A, None, None) == 4
    assert p(A, A, A, 32, 100, 4, A, None, None) == 2
    g = lq.lib.lutq_gemv_typed
    ws = lq.lutq_workspace_bytes(1, 64, 256, 4)

    def call(**kw):
        a = dict(dict(x=A, m=1, p=A, c=A, t=2, bits=4, n=64, k=256, y=A, ws=A, wsb=ws), **kw)
        return g(a["x"], a["m"], a["p"], a["c"], a["t"], a["bits"], a["n"], a["k"], a["y"],
                 a["ws"], a["wsb"], None, None)

    assert call(t=0) == 1
    assert call(t=5) == 1
    assert call(bits=3, t=3) == 1
    assert call(m=17) == 2                     # lutq_gemv's batch range
    assert call(m=0) == 2
    assert call(c=A + 8) == 4
    assert call(x=None) == 1
    gg = lq.lib.lutq_gemm_typed
    assert gg(A, 1, A, A, 0, 4, 64, 256, A, A, ws, None, None) == 1
    assert gg(A, 1, A, A, 3, 3, 64, 256, A, A, ws, None, None) == 1
    assert gg(A, 1, A, A, 2, 4, 64, 200, A, A, ws, None, None) == 2


def test_asym_linear_codebook_bit_exact_vs_oracle(lq):
    for lo, hi, bits in [(-0.5, 1.0, 4), (-2.0, 0.5, 3), (-0.031, 0.027, 4), (0.0, 0.0, 4),
                         (0.125, 0.5, 4)]:
        got = lq.lutq_codebook_asym_linear(lo, hi, bits).view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(got, O.bf16_bits(O.asym_linear_levels(lo, hi, bits)))
    f = lq.lib.lutq_codebook_asym_linear
    buf = (ctypes.c_uint16 * 16)()
    assert f(1.0, -1.0, 4, buf) == 1
    assert f(-1.0, 1.0, 5, buf) == 3
    assert f(float("nan"), 1.0, 4, buf) == 1
    assert f(-1.0, 1.0, 4, None) == 1


def test_group256_needs_k_multiple_of_256(lq):
    f = lq.lib.lutq_quantize_group256
    assert f(A, 32, 384, A, 4, A, A, None, None) == 2
    assert f(A, 32, 128, A, 4, A, A, None, None) == 2


def test_group64_sizes_and_argument_errors(lq):
    for n, k, bits in [(4096, 14336, 4), (4096, 4096, 3), (32, 128, 4)]:
        assert lq.lutq_packed_bytes_group64(n, k, bits) == \
            lq.lutq_packed_bytes(n, k, bits) + (n // 32) * (k // 128) * 64
    assert lq.lutq_packed_bytes_group64(33, 128, 4) == -1
    assert lq.lutq_packed_bytes_group64(32, 128, 2) == -1
    q, p = lq.lib.lutq_quantize_group64, lq.lib.lutq_pack_group64
    assert q(None, 32, 128, A, 4, A, A, None, None) == 1
    assert q(A, 32, 100, A, 4, A, A, None, None) == 2
    assert q(A, 32, 128, A, 5, A, A, None, None) == 3
    assert q(A, 32, 128, A, 4, A, A + 2, None, None) == 4
    assert p(None, A, 32, 128, 4, A, None, None) == 1
    assert p(A, A, 40, 128, 4, A, None, None) == 2
    assert p(A, A + 2, 32, 128, 4, A, None, None) == 4


def _variant_lib(name):
    path = os.path.join(ROOT, "dequant_gemv_group_b200", f"liblutq_{name}.so")
    if not os.path.exists(path):
        pytest.skip(f"liblutq_{name}.so is not built")
    return ctypes.CDLL(path)


def test_build_flags_of_each_build(lq):
    # the product build has neither tooling option; the variants one each,
    # and export the same functions
    assert lq.lutq_build_flags() == 0
    declared = _header_functions()
    for name, flag in (("nvtx", lq.BUILD_NVTX), ("bounds", lq.BUILD_BOUNDS)):
        lib = _variant_lib(name)
        assert lib.lutq_build_flags() == flag
        for fn in declared:
            assert hasattr(lib, fn), (name, fn)


def test_selftest_bounds_argument_error(lq):
    assert lq.lib.lutq_selftest_bounds(None, None) == 1
