"""Randomized Hadamard rotation on the GPU against the oracle (through the C
ABI): the rotated weights bit for bit (they decide the codes), the rotated
activations within one bf16 step (summed in fp32), the product with the
rotation fused into the GEMV's prologue bit for bit against the unfused
sequence, and within the 2e-3 gate against the oracle's rotated product."""
import numpy as np
import pytest
import torch

import workloads
from oracle import lutq_oracle as O

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def lq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import dequant_gemv_group_b200 as m
    return m


def _bits16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _f32(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("n,k", [(32, 128), (96, 640), (1024, 4096), (7, 1152)])
def test_rotations_match_oracle(lq, n, k):
    w = workloads.normal_weights(max(n, 32), k, 0.02, seed=n + k, outlier_frac=1e-2)[:n].contiguous()
    x = workloads.activations(n, k, seed=3)
    signs = workloads.rht_signs(7)
    wr = lq.lutq_rht_weights(w.cuda(), signs.cuda())
    xr = lq.lutq_rht_activations(x.cuda(), signs.cuda())
    torch.cuda.synchronize()
    # weights (they decide the codes): bit for bit with the oracle's exact sums
    want_w = O.bf16_bits(O.rht_weights(_f32(w), signs.numpy()))
    np.testing.assert_array_equal(_bits16(wr), want_w)
    # activations (an input of the fp32 product, summed in fp32): within one
    # bf16 step of the exactly rounded value, and exact for most entries
    want_x = O.rht_activations(_f32(x), signs.numpy())
    got_x = _f32(xr).astype(np.float64)
    step = np.abs(want_x) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(got_x - want_x) <= step)
    assert np.mean(got_x == want_x) > 0.95


def _rotated_layer(lq, w_cpu, signs, kind, bits):
    cb = lq.lutq_codebook(kind, bits)
    _, levels = O.codebook(kind, bits)
    wr = lq.lutq_rht_weights(w_cpu.cuda(), signs.cuda())
    st = lq.new_status()
    codes, scales = lq.lutq_quantize(wr, cb.cuda(), bits, status=st)
    packed = lq.lutq_pack(codes, scales, bits, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return cb.cuda(), levels, wr, codes, packed


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
@pytest.mark.parametrize("m", [1, 2, 3, 4])
@pytest.mark.parametrize("n,k", [(96, 1152), (1024, 4096), (320, 4224)])
def test_gemv_rht_fused_equals_unfused_and_oracle(lq, kind, bits, m, n, k):
    w = workloads.normal_weights(n, k, 0.02, seed=17 + n, outlier_frac=1e-3)
    x = workloads.activations(m, k, seed=19 + m)
    signs = workloads.rht_signs(23)
    cb, levels, wr, codes, packed = _rotated_layer(lq, w, signs, kind, bits)
    ws = lq.new_workspace(m, n, k, bits)
    st = lq.new_status()
    y_fused = lq.lutq_gemv_rht(x.cuda(), packed, cb, signs.cuda(), bits, n, k, workspace=ws,
                               status=st)
    xr = lq.lutq_rht_activations(x.cuda(), signs.cuda())
    y_plain = lq.lutq_gemv(xr, packed, cb, bits, n, k, workspace=ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(y_fused.cpu().numpy(), y_plain.cpu().numpy())
    # the oracle's pipeline: rotate, quantize, rotate x, product
    wr_ref = O.rht_weights(_f32(w), signs.numpy())
    np.testing.assert_array_equal(_bits16(wr), O.bf16_bits(wr_ref))
    ref_codes, ref_sb = O.quantize(wr_ref.astype(np.float32), levels, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    xr_ref = O.rht_activations(_f32(x), signs.numpy())
    y_ref = O.gemv(xr_ref, ref_codes, ref_sb, levels)
    assert O.rel_error_gate(y_fused.cpu().numpy(), y_ref) <= TOL


def test_gemv_rht_full_size_layer(lq):
    lay = workloads.layer("llama3_8b_w4_nf4", "down")
    n, k = lay.n, lay.k
    w = lay.weights(seed=0)
    signs = workloads.rht_signs(29)
    cb, levels, wr, codes, packed = _rotated_layer(lq, w, signs, "nf4", 4)
    x = workloads.activations(1, k, seed=1)
    y = lq.lutq_gemv_rht(x.cuda(), packed, cb, signs.cuda(), 4, n, k,
                         workspace=lq.new_workspace(1, n, k, 4))
    torch.cuda.synchronize()
    strips = [0, 17, 127]
    rows = np.concatenate([np.arange(32 * s, 32 * s + 32) for s in strips])
    wr_ref = O.rht_weights(_f32(w[rows]), signs.numpy())
    ref_codes, ref_sb = O.quantize(wr_ref.astype(np.float32), levels, 4)
    np.testing.assert_array_equal(codes[rows].cpu().numpy(), ref_codes)
    y_ref = O.gemv(O.rht_activations(_f32(x), signs.numpy()), ref_codes, ref_sb, levels)
    assert O.rel_error_gate(y.cpu().numpy()[:, rows], y_ref) <= TOL


def test_rotation_lowers_the_products_error_on_the_gpu(lq):
    # the method's purpose, end to end through the library: with 1% outliers
    # the rotated product is closer to the unquantized one
    n, k, m = 512, 4096, 2
    w = workloads.normal_weights(n, k, 0.02, seed=31, outlier_frac=1e-2)
    x = workloads.activations(m, k, seed=32)
    signs = workloads.rht_signs(33)
    exact = _f32(x).astype(np.float64) @ _f32(w).astype(np.float64).T
    cb = lq.lutq_codebook("nf4", 4).cuda()
    codes, scales = lq.lutq_quantize(w.cuda(), cb, 4)
    y0 = lq.lutq_gemv(x.cuda(), lq.lutq_pack(codes, scales, 4), cb, 4, n, k,
                      workspace=lq.new_workspace(m, n, k, 4))
    _, _, _, _, packed_r = _rotated_layer(lq, w, signs, "nf4", 4)
    y1 = lq.lutq_gemv_rht(x.cuda(), packed_r, cb, signs.cuda(), 4, n, k,
                          workspace=lq.new_workspace(m, n, k, 4))
    torch.cuda.synchronize()
    e0 = np.linalg.norm(y0.cpu().numpy() - exact)
    e1 = np.linalg.norm(y1.cpu().numpy() - exact)
    assert e1 < 0.9 * e0
