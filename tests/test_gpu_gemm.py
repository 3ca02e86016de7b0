"""Parity of the tensor-core product (lutq_gemm, tcgen05) with the CPU oracle.

Same gate as the GEMV: y within 2e-3 (relative, floored at 1e-2 of the row
rms) of the fp64 oracle; one-hot inputs reproduce the dequantized weights
exactly; repeated calls are bitwise identical.  Shapes cover partial row
tiles (N not a multiple of 128), several groups, batch sizes that are not a
multiple of 16 and more than one 128-wide batch tile.
"""
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


def _prep(lq, w, kind, bits):
    cb = lq.lutq_codebook(kind, bits).cuda()
    st = lq.new_status()
    codes, scales = lq.lutq_quantize(w.cuda(), cb, bits, status=st)
    packed = lq.lutq_pack(codes, scales, bits, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return cb, codes, scales, packed


def _gemm(lq, x, packed, scales, cb, bits, n, k, ws=None):
    m = x.shape[0]
    if ws is None:
        ws = lq.new_workspace(m, n, k, bits)
    st = lq.new_status()
    y = lq.lutq_gemm(x.cuda(), packed, cb, bits, n, k, workspace=ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, lq.lutq_status_string(int(st.item()))
    return y.cpu().numpy(), ws


def _bits16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
@pytest.mark.parametrize("m", [1, 5, 16, 17, 32, 48, 64, 100, 128, 130])
@pytest.mark.parametrize("n,k", [(32, 128), (96, 1152), (256, 640), (1024, 2048)])
def test_gemm_small_full_compare(lq, kind, bits, m, n, k):
    w = workloads.normal_weights(n, k, 0.02, seed=n + 3 * k, outlier_frac=1e-3)
    cb, codes, scales, packed = _prep(lq, w, kind, bits)
    _, levels = O.codebook(kind, bits)
    ref_codes, ref_sb = O.quantize(w.float().numpy(), levels, bits)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    x = workloads.activations(m, k, seed=m)
    y, ws = _gemm(lq, x, packed, scales, cb, bits, n, k)
    y_ref = O.gemv(x.float().numpy(), ref_codes, ref_sb, levels)
    assert O.rel_error_gate(y, y_ref) <= TOL
    # the per-strip arrival counters at the start of the workspace are back to zero
    n_counters = -(-m // 128) * -(-n // 128) * 4 * 2
    assert int(ws.view(torch.int32)[:n_counters].abs().sum().item()) == 0


@pytest.mark.parametrize("bits,kind", [(4, "logb"), (3, "lloyd_max3")])
def test_gemm_one_hot_is_exact(lq, bits, kind):
    n, k = 160, 384
    w = workloads.student_t_weights(n, k, 5, 0.02, seed=2)
    cb, codes, scales, packed = _prep(lq, w, kind, bits)
    _, levels = O.codebook(kind, bits)
    wh = O.dequant(codes.cpu().numpy(), _bits16(scales), levels)
    ks = list(range(0, 384, 7))[:40]
    x = torch.zeros((len(ks), k), dtype=torch.bfloat16)
    for i, kk in enumerate(ks):
        x[i, kk] = 1.0
    y, _ = _gemm(lq, x, packed, scales, cb, bits, n, k)
    for i, kk in enumerate(ks):
        np.testing.assert_array_equal(y[i].astype(np.float64), wh[:, kk])


def test_gemm_deterministic_and_agrees_with_gemv(lq):
    n, k = 4096, 4096
    w = workloads.normal_weights(n, k, 0.02, seed=9)
    cb, codes, scales, packed = _prep(lq, w, "nf4", 4)
    x = workloads.activations(16, k, seed=10)
    y1, ws = _gemm(lq, x, packed, scales, cb, 4, n, k)
    y2, _ = _gemm(lq, x, packed, scales, cb, 4, n, k, ws=ws)
    np.testing.assert_array_equal(y1, y2)
    st = lq.new_status()
    yv = lq.lutq_gemv(x.cuda(), packed, cb, 4, n, k, workspace=ws, status=st)
    torch.cuda.synchronize()
    assert O.rel_error_gate(y1, yv.cpu().numpy().astype(np.float64)) <= TOL


@pytest.mark.parametrize("layer", ["gate_up", "down"])
@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
def test_workload_70b_gemm(lq, layer, kind, bits):
    lay = workloads.layer("llama3_70b_mlp", layer)
    n, k = lay.n, lay.k
    w = lay.weights(seed=0)
    cb, codes, scales, packed = _prep(lq, w, kind, bits)
    rng = np.random.default_rng(1)
    strips = sorted({0, n // 32 - 1} | set(rng.integers(0, n // 32, size=3).tolist()))
    rows = np.concatenate([np.arange(32 * s, 32 * s + 32) for s in strips])
    _, levels = O.codebook(kind, bits)
    ref_codes, ref_sb = O.quantize(w[rows].float().numpy(), levels, bits)
    assert np.array_equal(codes[rows].cpu().numpy(), ref_codes)
    del w
    ws = lq.new_workspace(128, n, k, bits)
    # batches between the GEMV's 16 and 32 take the 32-wide batch tile with
    # its rows past M read as zero: 24 and 31 are ragged ones
    for m in (24, 31, 32, 64, 128):
        x = workloads.activations(m, k, seed=1)
        y, _ = _gemm(lq, x, packed, scales, cb, bits, n, k, ws=ws)
        y_ref = O.gemv(x.float().numpy(), ref_codes, ref_sb, levels)
        assert O.rel_error_gate(y[:, rows], y_ref) <= TOL, (layer, kind, m)
