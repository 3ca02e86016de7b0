"""One scale per group of 64 on the GPU against the oracle (through the C ABI).

Codes, scales [N, K/64] and the packed bytes (128-byte scale blocks) must
match the oracle's quantize_group64 / pack_group64 bit for bit, and the
packing must reproduce the hand-derived scale bytes of
tests/golden/pack_v2_scales_group64.txt.  y from the CUDA-core GEMV and the
tensor-core GEMM must lie within the 2e-3 relative gate of the oracle's fp64
gemv_group64.  Small cases are compared in full; one full-size layer on
sampled 32-row strips.
"""
import os

import numpy as np
import pytest
import torch

import workloads
from oracle import lutq_oracle as O

pytestmark = pytest.mark.gpu

TOL = 2e-3
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def lq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import dequant_gemv_group_b200 as m
    return m


def _f32(t):
    return t.float().cpu().numpy()


def _bits16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _weights(n, k, seed):
    w = workloads.normal_weights(n, k, 0.02, seed=seed, outlier_frac=1e-3)
    if n > 3:
        w[3] = 0.0                     # an all-zero row
    if n > 5 and k >= 128:
        w[5, 64:128] = 0.0             # a zero 64-group beside a non-zero one
        w[5, 0] = 1.0                  # and a large weight in its neighbour
    return w


def _quantize_pack(lq, w, kind, bits):
    cb = lq.lutq_codebook(kind, bits).cuda()
    _, levels = O.codebook(kind, bits)
    st = lq.new_status()
    codes, scales = lq.lutq_quantize_group64(w.cuda(), cb, bits, status=st)
    packed = lq.lutq_pack_group64(codes, scales, bits, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return cb, levels, codes, scales, packed


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("logb", 4), ("lloyd_max3", 3)])
@pytest.mark.parametrize("n,k", [(32, 128), (96, 640), (256, 1024)])
def test_quantize_and_pack_bit_exact(lq, kind, bits, n, k):
    w = _weights(n, k, seed=n + k + bits)
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, kind, bits)
    rc, rs = O.quantize_group64(_f32(w), levels, bits)
    assert tuple(scales.shape) == (n, k // 64)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(_bits16(scales), rs)
    assert packed.numel() == lq.lutq_packed_bytes_group64(n, k, bits)
    np.testing.assert_array_equal(packed.cpu().numpy(), O.pack_group64(rc, rs, bits))


def test_pack_hand_derived_scale_bytes(lq):
    n, k = 64, 256
    nn, hh = np.meshgrid(np.arange(n), np.arange(4), indexing="ij")
    sb = (0x3C00 + 8 * nn + hh).astype(np.uint16)
    scales = torch.from_numpy(sb.view(np.int16)).view(torch.bfloat16).cuda()
    codes = torch.zeros((n, k), dtype=torch.uint8, device="cuda")
    pk = lq.lutq_pack_group64(codes, scales, 4).cpu().numpy()
    seen = 0
    with open(os.path.join(GOLDEN, "pack_v2_scales_group64.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            off = int(parts[0])
            assert bytes(pk[off:off + 2]) == bytes(int(b, 16) for b in parts[1:]), off
            seen += 1
    assert seen == 5


def test_quantize_reports_nonfinite(lq):
    w = _weights(64, 256, seed=1)
    w[40, 70] = float("inf")
    cb = lq.lutq_codebook("nf4", 4).cuda()
    st = lq.new_status()
    lq.lutq_quantize_group64(w.cuda(), cb, 4, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5


# shapes that select each GEMV work plan (whole strips, unit ranges,
# main/helper blocks), a ragged last row tile for the tensor-core kernel, and
# batches on both kernels
@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
@pytest.mark.parametrize("n,k", [(96, 1152), (1024, 4096), (256, 14336), (320, 4224)])
def test_gemv_and_gemm_against_oracle(lq, kind, bits, n, k):
    w = _weights(n, k, seed=7 * n + bits)
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, kind, bits)
    rc, rs = O.quantize_group64(_f32(w), levels, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(_bits16(scales), rs)
    ws = lq.new_workspace(200, n, k, bits)
    st = lq.new_status()
    for m in (1, 2, 3, 4, 8, 16, 24, 64, 200):
        x = workloads.activations(m, k, seed=m)
        y_ref = O.gemv_group64(_f32(x), rc, rs, levels)
        fns = [lq.lutq_gemv_group64] if m <= 16 else []
        if m in (1, 16, 24, 64, 200):
            fns.append(lq.lutq_gemm_group64)
        for fn in fns:
            y = fn(x.cuda(), packed, cb, bits, n, k, workspace=ws, status=st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0, (fn.__name__, m)
            assert O.rel_error_gate(y.cpu().numpy(), y_ref) <= TOL, (fn.__name__, m)


def test_group64_differs_from_group128(lq):
    # the two 64-halves of each group carry their own scales: reading the
    # 128-byte blocks as one scale per group would fail the gate
    n, k, bits = 256, 1024, 4
    w = workloads.normal_weights(n, k, 0.02, seed=11, outlier_frac=1e-2)
    w[:, 64::128] *= 8.0               # make the second halves' maxima differ
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, "nf4", bits)
    rc, rs = O.quantize_group64(_f32(w), levels, bits)
    x = workloads.activations(1, k, seed=3)
    y = lq.lutq_gemv_group64(x.cuda(), packed, cb, bits, n, k,
                             workspace=lq.new_workspace(1, n, k, bits))
    torch.cuda.synchronize()
    y_ref = O.gemv_group64(_f32(x), rc, rs, levels)
    assert O.rel_error_gate(y.cpu().numpy(), y_ref) <= TOL
    s128 = np.maximum(rs[:, 0::2], rs[:, 1::2])            # bf16 bits order as magnitudes
    y_wrong = O.gemv(_f32(x), rc, s128, levels)
    assert O.rel_error_gate(y_wrong, y_ref) > 10 * TOL


def _sample_strips(n, count=3, seed=0):
    strips = n // 32
    rng = np.random.default_rng(seed)
    pick = {0, strips - 1} | set(rng.integers(0, strips, size=count).tolist())
    return sorted(pick)


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
def test_full_size_layer_sampled(lq, kind, bits):
    lay = workloads.layer("llama3_8b_w4_nf4", "down")
    n, k = lay.n, lay.k
    w = lay.weights(seed=0)
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, kind, bits)
    strips = _sample_strips(n)
    rows = np.concatenate([np.arange(32 * s, 32 * s + 32) for s in strips])
    rc, rs = O.quantize_group64(_f32(w[rows]), levels, bits)
    np.testing.assert_array_equal(codes[rows].cpu().numpy(), rc)
    np.testing.assert_array_equal(_bits16(scales[rows]), rs)
    tb = 2048 if bits == 4 else 1536
    g = k // 128
    units = (n // 32) * g
    pk = packed.cpu().numpy()
    for i, s in enumerate(strips):
        want = O.pack_group64(rc[32 * i: 32 * i + 32], rs[32 * i: 32 * i + 32], bits)
        np.testing.assert_array_equal(pk[s * g * tb:(s + 1) * g * tb], want[:g * tb])
        sc0 = units * tb + s * g * 128
        np.testing.assert_array_equal(pk[sc0:sc0 + g * 128], want[g * tb:])
    del w
    ws = lq.new_workspace(64, n, k, bits)
    st = lq.new_status()
    for m, fn in ((1, lq.lutq_gemv_group64), (4, lq.lutq_gemv_group64),
                  (16, lq.lutq_gemv_group64), (64, lq.lutq_gemm_group64)):
        x = workloads.activations(m, k, seed=1)
        y = fn(x.cuda(), packed, cb, bits, n, k, workspace=ws, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        y_ref = O.gemv_group64(_f32(x), rc, rs, levels)
        assert O.rel_error_gate(y.cpu().numpy()[:, rows], y_ref) <= TOL, (kind, m)
