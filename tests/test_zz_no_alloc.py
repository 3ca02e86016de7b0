"""lutq_gemv_noalloc: the GEMV for callers that cannot allocate device memory
where they run it (graph capture in a mode where cudaMalloc is illegal,
latency-critical loops that must not block in cudaMalloc, plug-in hosts
without an allocator).

It must give the same products as lutq_gemv (with a caller workspace), and
agree with the oracle, within the tolerance the GEMV tests use, on two calls
in a row, because every call shares the library's fixed scratch array and must
not depend on what the previous call left there.  It is called through the C
ABI directly.  This file is collected last so that a run stopping at the first
failure has run every other test; it passes alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import lutq_oracle as O

TOL = 2e-3
ARRAY_ZERO_BYTES = 1 << 20      # the array's zero part
ARRAY_SCRATCH_BYTES = 7 << 20   # and its scratch


@pytest.fixture(scope="module")
def lq():
    import dequant_gemv_group_b200 as m
    return m


def _f32(t):
    return t.float().cpu().numpy()


def _bits16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.gpu
@pytest.mark.parametrize("n,k,bits,kind,m", [(4096, 4096, 4, "nf4", 1),
                                             (1024, 14336, 3, "lloyd_max3", 4),
                                             (96, 1152, 4, "logb", 16)])
def test_noalloc_matches_workspace_gemv_and_oracle_twice(lq, n, k, bits, kind, m):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = workloads.normal_weights(n, k, 0.02, seed=21, outlier_frac=1e-3)
    cb = lq.lutq_codebook(kind, bits).cuda()
    _, levels = O.codebook(kind, bits)
    codes, scales = lq.lutq_quantize(w.cuda(), cb, bits)
    packed = lq.lutq_pack(codes, scales, bits)
    # the oracle's own quantization of the first rows, checked against the GPU's
    rows = np.arange(min(n, 256))
    rc, rs = O.quantize(_f32(w[rows]), levels, bits)
    np.testing.assert_array_equal(codes[rows].cpu().numpy(), rc)
    np.testing.assert_array_equal(_bits16(scales[rows]), rs)
    x = workloads.activations(m, k, seed=22)
    y_oracle = O.gemv(_f32(x), rc, rs, levels)
    x = x.cuda()
    ws = lq.new_workspace(m, n, k, bits)
    y_ref = lq.lutq_gemv(x, packed, cb, bits, n, k, workspace=ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
        st = lq.new_status()
        rc_ = lq.lib.lutq_gemv_noalloc(x.data_ptr(), m, packed.data_ptr(), cb.data_ptr(), bits,
                                       n, k, y.data_ptr(), st.data_ptr(), stream)
        torch.cuda.synchronize()
        assert rc_ == 0, lq.lutq_status_string(rc_)
        assert int(st.item()) == 0
        yh = y.cpu().numpy()
        assert O.rel_error_gate(yh, y_ref.cpu().numpy().astype(np.float64)) <= TOL
        assert O.rel_error_gate(yh[:, rows], y_oracle) <= TOL


def test_noalloc_rejects_problems_beyond_its_array(lq):
    # 2^26 rows need 32 N = 2 GiB of zero-at-start slots: more than the 1 MiB
    # part.  The size check comes before any device work, so aligned
    # placeholder addresses are never touched.
    a = 1 << 20
    rc = lq.lib.lutq_gemv_noalloc(a, 1, a, a, 4, 1 << 26, 128, a, None, None)
    assert rc == 9


@pytest.mark.parametrize("m", list(range(5, 17)))
def test_noalloc_bound_for_batches_5_to_16(lq, m):
    # The call is rejected exactly when the problem's zero part exceeds the
    # array's 1 MiB or its tensor-core scratch exceeds the other 7 MiB,
    # whichever kernel would run it.  Only rejected shapes are called when a
    # GPU is present (placeholder addresses never reach a kernel); without
    # one, an accepted shape fails later, at the CUDA set-up.
    a = 1 << 20
    gpu = torch.cuda.is_available()
    for n in (32, 4096, 32768, 32800, 65536):
        for k, bits in ((128, 4), (14336, 3)):
            zero = lq.lutq_workspace_zero_bytes(m, n, k, bits)
            scratch = lq.lutq_workspace_bytes(m, n, k, bits) - zero
            rejected = zero > ARRAY_ZERO_BYTES or scratch > ARRAY_SCRATCH_BYTES
            assert rejected == (n > 32768), (m, n, k, zero, scratch)
            if rejected:
                assert lq.lib.lutq_gemv_noalloc(a, m, a, a, bits, n, k, a, None, None) == 9
            elif not gpu:
                assert lq.lib.lutq_gemv_noalloc(a, m, a, a, bits, n, k, a, None, None) == 8
