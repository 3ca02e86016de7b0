"""The layer histogram on the GPU (lutq_fit_histogram) against the oracle's,
count for count, and a fitted codebook through the whole path: its codes,
scales and product match the oracle and its product error is lower than the
starting codebook's."""
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


@pytest.mark.parametrize("n,k", [(32, 128), (96, 1152), (1024, 4096), (5, 384)])
def test_histogram_counts_match_oracle(lq, n, k):
    w = workloads.student_t_weights(max(n, 32), k, 5, 0.02, seed=n, outlier_frac=1e-2)[:n]
    w = w.contiguous()
    w[0, :128] = 0.0                       # an all-zero group
    w[-1, 5] = -0.0
    h = lq.lutq_fit_histogram(w.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(h.cpu().numpy(), O.fit_histogram(w.float().numpy()))


def test_histogram_accumulates_and_reports_nonfinite(lq):
    a = workloads.normal_weights(64, 512, 0.02, seed=1)
    b = workloads.normal_weights(32, 512, 0.02, seed=2)
    h = lq.lutq_fit_histogram(a.cuda())
    lq.lutq_fit_histogram(b.cuda(), hist=h)
    torch.cuda.synchronize()
    want = O.fit_histogram(a.float().numpy()) + O.fit_histogram(b.float().numpy())
    np.testing.assert_array_equal(h.cpu().numpy(), want)
    bad = a.clone()
    bad[3, 7] = float("nan")
    st = lq.new_status()
    lq.lutq_fit_histogram(bad.cuda(), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
def test_fitted_codebook_through_the_path(lq, kind, bits):
    n, k, m = 1024, 4096, 2
    w = workloads.student_t_weights(n, k, 5, 0.02, seed=7, outlier_frac=1e-3)
    x = workloads.activations(m, k, seed=8)
    h = lq.lutq_fit_histogram(w.cuda())
    init = lq.lutq_codebook(kind, bits)
    fitted = lq.lutq_fit_codebook(h.cpu(), bits, init)
    # the oracle's fit of the oracle's histogram
    _, init_lv = O.codebook(kind, bits)
    want = O.fit_codebook(O.fit_histogram(w.float().numpy()), init_lv)
    np.testing.assert_array_equal(fitted.view(torch.int16).numpy().view(np.uint16),
                                  O.bf16_bits(want))
    levels = want.astype(np.float32)
    st = lq.new_status()
    codes, scales = lq.lutq_quantize(w.cuda(), fitted.cuda(), bits, status=st)
    packed = lq.lutq_pack(codes, scales, bits, status=st)
    y = lq.lutq_gemv(x.cuda(), packed, fitted.cuda(), bits, n, k,
                     workspace=lq.new_workspace(m, n, k, bits), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref_codes, ref_sb = O.quantize(w.float().numpy(), levels, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    y_ref = O.gemv(x.float().numpy(), ref_codes, ref_sb, levels)
    assert O.rel_error_gate(y.cpu().numpy(), y_ref) <= TOL
    # lower product error than the starting codebook
    exact = x.double().numpy() @ w.double().numpy().T
    c0, s0 = O.quantize(w.float().numpy(), init_lv, bits)
    e0 = np.linalg.norm(O.gemv(x.float().numpy(), c0, s0, init_lv) - exact)
    e1 = np.linalg.norm(y_ref - exact)
    assert e1 < e0
