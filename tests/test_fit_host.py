"""The library's host-side codebook fitting (lutq_fit_codebook, C++) against
the oracle's, bit for bit, on histograms with known and with realistic
shapes; no GPU is involved."""
import numpy as np
import pytest
import torch

import workloads
from oracle import lutq_oracle as O


@pytest.fixture(scope="module")
def lq():
    import dequant_gemv_group_b200 as m
    return m


def _bits(levels):
    return O.bf16_bits(levels)


def _lib_fit(lq, hist, bits, init_bits, max_iter=100):
    h = np.ascontiguousarray(np.asarray(hist, dtype=np.uint64))
    init = np.ascontiguousarray(np.asarray(init_bits, dtype=np.uint16))
    out = np.zeros(1 << bits, dtype=np.uint16)
    rc = lq.lib.lutq_fit_codebook(h.ctypes.data, bits, init.ctypes.data, max_iter, out.ctypes.data)
    assert rc == 0, lq.lutq_status_string(rc)
    return out


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3), ("logb", 4),
                                       ("uniform4", 4)])
def test_fit_matches_oracle_on_layer_histograms(lq, kind, bits):
    w = workloads.student_t_weights(256, 2048, 5, 0.02, seed=40 + bits, outlier_frac=1e-3)
    h = O.fit_histogram(w.float().numpy())
    init_bits, init = O.codebook(kind, bits)
    want = O.fit_codebook(h, init)
    np.testing.assert_array_equal(_lib_fit(lq, h, bits, init_bits), _bits(want))


def test_fit_matches_oracle_on_random_and_sparse_histograms(lq):
    rng = np.random.default_rng(5)
    init_bits, init = O.codebook("nf4", 4)
    for trial in range(4):
        h = np.zeros(O.HIST_BINS, np.int64)
        idx = rng.integers(0, O.HIST_BINS, size=50 * (trial + 1))
        np.add.at(h, idx, rng.integers(1, 1000, size=idx.size))
        for it in (1, 3, 100):
            np.testing.assert_array_equal(_lib_fit(lq, h, 4, init_bits, it),
                                          _bits(O.fit_codebook(h, init, it)))


def test_fit_zero_iterations_returns_the_start(lq):
    init_bits, _ = O.codebook("nf4", 4)
    h = np.ones(O.HIST_BINS, np.int64)
    np.testing.assert_array_equal(_lib_fit(lq, h, 4, init_bits, 0), init_bits)


def test_fit_codebook_argument_errors(lq):
    f = lq.lib.lutq_fit_codebook
    h = np.zeros(O.HIST_BINS, np.uint64)
    init = np.zeros(16, np.uint16)
    out = np.zeros(16, np.uint16)
    assert f(None, 4, init.ctypes.data, 10, out.ctypes.data) == 1
    assert f(h.ctypes.data, 5, init.ctypes.data, 10, out.ctypes.data) == 3
    assert f(h.ctypes.data, 4, init.ctypes.data, -1, out.ctypes.data) == 1
    big = h.copy()
    big[0] = 1 << 31
    assert f(big.ctypes.data, 4, init.ctypes.data, 10, out.ctypes.data) == 1


def test_binding_wrapper(lq):
    w = workloads.normal_weights(64, 1024, 0.02, seed=3, outlier_frac=1e-3)
    h = O.fit_histogram(w.float().numpy())
    init = lq.lutq_codebook("nf4", 4)
    got = lq.lutq_fit_codebook(torch.from_numpy(h), 4, init)
    _, lv = O.codebook("nf4", 4)
    np.testing.assert_array_equal(got.view(torch.int16).numpy().view(np.uint16),
                                  _bits(O.fit_codebook(h, lv)))
