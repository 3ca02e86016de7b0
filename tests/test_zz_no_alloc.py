"""lutq_gemv_noalloc: the GEMV for callers that cannot allocate device memory.

It must give the same products as lutq_gemv (with a caller workspace), within
the tolerance the GEMV tests use, on two calls in a row, because every call
shares the library's fixed scratch array and must not depend on what the
previous call left there.  It is called through the C ABI directly.  This
file is collected last so that a run stopping at the first failure has run
every other test; it passes alone in a fresh process as well.
"""
import ctypes

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


@pytest.mark.parametrize("n,k,bits,kind,m", [(4096, 4096, 4, "nf4", 1),
                                             (1024, 14336, 3, "lloyd_max3", 4),
                                             (96, 1152, 4, "logb", 16)])
def test_noalloc_matches_workspace_gemv_twice(lq, n, k, bits, kind, m):
    w = workloads.normal_weights(n, k, 0.02, seed=21, outlier_frac=1e-3).cuda()
    cb = lq.lutq_codebook(kind, bits).cuda()
    codes, scales = lq.lutq_quantize(w, cb, bits)
    packed = lq.lutq_pack(codes, scales, bits)
    x = workloads.activations(m, k, seed=22).cuda()
    ws = lq.new_workspace(m, n, k, bits)
    y_ref = lq.lutq_gemv(x, packed, cb, bits, n, k, workspace=ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
        st = lq.new_status()
        rc = lq.lib.lutq_gemv_noalloc(x.data_ptr(), m, packed.data_ptr(), cb.data_ptr(), bits,
                                      n, k, y.data_ptr(), st.data_ptr(), stream)
        torch.cuda.synchronize()
        assert rc == 0, lq.lutq_status_string(rc)
        assert int(st.item()) == 0
        assert O.rel_error_gate(y.cpu().numpy(), y_ref.cpu().numpy().astype(np.float64)) <= TOL


def test_noalloc_rejects_problems_beyond_its_array(lq):
    # 2^26 rows need 8 N = 512 MiB of exchange slots: more than the 4 MiB array.  The
    # size check comes before any device work, so aligned placeholder
    # addresses are never touched.
    a = 1 << 20
    rc = lq.lib.lutq_gemv_noalloc(a, 1, a, a, 4, 1 << 26, 128, a, None, None)
    assert rc == 9
