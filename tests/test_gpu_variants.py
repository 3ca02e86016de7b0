"""Format variants on the GPU against the oracle (through the C ABI): one
scale per row (codes and scales bit for bit, the product within the gate),
and the bf16 output of the products (bit for bit the fp32 output rounded once
to bf16, within the gate widened by one bf16 rounding against the oracle)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import lutq_oracle as O

pytestmark = pytest.mark.gpu

TOL = 2e-3
TOL_BF16 = 2e-3 + 2.0 ** -9      # the fp32 gate plus one bf16 rounding of y


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


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("logb", 4), ("lloyd_max3", 3)])
@pytest.mark.parametrize("n,k", [(32, 128), (96, 1152), (1024, 4096), (64, 14336)])
def test_rowscale_quantize_bit_exact_and_product(lq, kind, bits, n, k):
    w = workloads.normal_weights(n, k, 0.02, seed=n + k, outlier_frac=1e-2)
    w[3] = 0.0                                        # an all-zero row
    cb = lq.lutq_codebook(kind, bits).cuda()
    _, levels = O.codebook(kind, bits)
    st = lq.new_status()
    codes, scales = lq.lutq_quantize_rowscale(w.cuda(), cb, bits, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rc, rs = O.quantize_rowscale(_f32(w), levels, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(_bits16(scales), rs)
    packed = lq.lutq_pack(codes, scales, bits, status=st)
    x = workloads.activations(2, k, seed=5)
    y = lq.lutq_gemv(x.cuda(), packed, cb, bits, n, k, workspace=lq.new_workspace(2, n, k, bits),
                     status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert O.rel_error_gate(y.cpu().numpy(), O.gemv(_f32(x), rc, rs, levels)) <= TOL


def _layer(lq, n, k, kind, bits, seed):
    w = workloads.normal_weights(n, k, 0.02, seed=seed, outlier_frac=1e-3)
    cb = lq.lutq_codebook(kind, bits).cuda()
    _, levels = O.codebook(kind, bits)
    codes, scales = lq.lutq_quantize(w.cuda(), cb, bits)
    packed = lq.lutq_pack(codes, scales, bits)
    # the oracle's own quantization of the first rows (at most 256), checked
    # against the GPU's: the product checks below take it as their reference
    rows = np.arange(min(n, 256))
    rc, rs = O.quantize(_f32(w[rows]), levels, bits)
    np.testing.assert_array_equal(codes[rows].cpu().numpy(), rc)
    np.testing.assert_array_equal(_bits16(scales[rows]), rs)
    return cb, levels, (rc, rs), packed


# shapes that select each GEMV work plan (whole strips, unit ranges,
# main/helper blocks) and the tensor-core kernel
@pytest.mark.parametrize("n,k,m", [(4096, 4096, 1), (14336, 4096, 2), (1024, 4096, 3),
                                   (256, 14336, 4), (1024, 4096, 8), (512, 2048, 32),
                                   (320, 4224, 128)])
@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
def test_bf16_output_is_the_fp32_output_rounded(lq, n, k, m, kind, bits):
    cb, levels, (rc, rs), packed = _layer(lq, n, k, kind, bits, seed=n + m)
    x = workloads.activations(m, k, seed=m).cuda()
    ws = lq.new_workspace(m, n, k, bits)
    st = lq.new_status()
    pairs = [(lq.lutq_gemv, lq.lutq_gemv_out_bf16)] if m <= 16 else []
    pairs.append((lq.lutq_gemm, lq.lutq_gemm_out_bf16))
    y_ref = None
    for f32_fn, bf16_fn in pairs:
        y32 = f32_fn(x, packed, cb, bits, n, k, workspace=ws, status=st)
        y16 = bf16_fn(x, packed, cb, bits, n, k, workspace=ws, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert y16.dtype == torch.bfloat16
        assert torch.equal(y16, y32.to(torch.bfloat16)), bf16_fn.__name__
        if y_ref is None:
            y_ref = O.gemv(_f32(x), rc, rs, levels)
        assert O.rel_error_gate(_f32(y16)[:, :y_ref.shape[1]], y_ref) <= TOL_BF16


@pytest.mark.parametrize("bits", [4, 3])
@pytest.mark.parametrize("n,k", [(96, 1152), (1024, 4096), (4096, 256)])
def test_tensorscale_asym_linear_bit_exact_and_product(lq, bits, n, k):
    # the tensor-wise asymmetric linear baseline: levels evenly spaced from
    # min W to max W over one scale for the matrix
    w = workloads.normal_weights(n, k, 0.02, seed=3 * n + bits, outlier_frac=1e-3)
    lo, hi = float(w.float().min()), float(w.float().max())
    cb = lq.lutq_codebook_asym_linear(lo, hi, bits)
    levels = O.asym_linear_levels(lo, hi, bits).astype(np.float32)
    np.testing.assert_array_equal(_bits16(cb), O.bf16_bits(levels))
    st = lq.new_status()
    codes, scales = lq.lutq_quantize_tensorscale(w.cuda(), cb.cuda(), bits, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rc, rs = O.quantize_tensorscale(_f32(w), levels, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(_bits16(scales), rs)
    x = workloads.activations(1, k, seed=9)
    y = lq.lutq_gemv(x.cuda(), lq.lutq_pack(codes, scales, bits), cb.cuda(), bits, n, k,
                     workspace=lq.new_workspace(1, n, k, bits), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert O.rel_error_gate(y.cpu().numpy(), O.gemv(_f32(x), rc, rs, levels)) <= TOL


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
@pytest.mark.parametrize("n,k", [(32, 256), (96, 1280), (1024, 4096)])
def test_group256_quantize_bit_exact_and_product(lq, kind, bits, n, k):
    w = workloads.normal_weights(n, k, 0.02, seed=7 * n + bits, outlier_frac=1e-2)
    w[5, 256:512] = 0.0                               # an all-zero 256-group
    cb = lq.lutq_codebook(kind, bits).cuda()
    _, levels = O.codebook(kind, bits)
    st = lq.new_status()
    codes, scales = lq.lutq_quantize_group256(w.cuda(), cb, bits, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rc, rs = O.quantize_group256(_f32(w), levels, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(_bits16(scales), rs)
    x = workloads.activations(3, k, seed=13)
    y = lq.lutq_gemv(x.cuda(), lq.lutq_pack(codes, scales, bits, status=st), cb, bits, n, k,
                     workspace=lq.new_workspace(3, n, k, bits), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert O.rel_error_gate(y.cpu().numpy(), O.gemv(_f32(x), rc, rs, levels)) <= TOL
