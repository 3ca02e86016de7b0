"""The bound on the kernels' pipeline waits: a wait on a barrier that nothing
completes ends by itself, reports LUTQ_ERR_TIMEOUT in the device status word,
and the context keeps working (a product launched after it is still exact)."""
import time

import numpy as np
import pytest
import torch

import workloads
from oracle import lutq_oracle as O

pytestmark = pytest.mark.gpu

LUTQ_ERR_TIMEOUT = 7
LUTQ_ERR_BITS = 3


@pytest.fixture(scope="module")
def lq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import dequant_gemv_group_b200 as m
    return m


def test_wait_runs_out_and_reports(lq):
    st = lq.new_status()
    t0 = time.perf_counter()
    lq.lutq_selftest_wait_timeout(st, 2_000_000)  # 2 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(st.item()) == LUTQ_ERR_TIMEOUT
    assert elapsed < 1.0
    # an earlier error in the word is kept (the first error wins)
    st2 = torch.full((1,), LUTQ_ERR_BITS, dtype=torch.int32, device="cuda")
    lq.lutq_selftest_wait_timeout(st2, 1_000_000)
    torch.cuda.synchronize()
    assert int(st2.item()) == LUTQ_ERR_BITS


def test_context_usable_after_timeout(lq):
    st = lq.new_status()
    lq.lutq_selftest_wait_timeout(st, 1_000_000)
    n, k, bits = 256, 1024, 4
    w = workloads.normal_weights(n, k, 0.02, seed=3)
    cb = lq.lutq_codebook("nf4", bits)
    _, levels = O.codebook("nf4", bits)
    st2 = lq.new_status()
    codes, scales = lq.lutq_quantize(w.cuda(), cb.cuda(), bits, status=st2)
    packed = lq.lutq_pack(codes, scales, bits, status=st2)
    x = workloads.activations(1, k, seed=4)
    y = lq.lutq_gemv(x.cuda(), packed, cb.cuda(), bits, n, k,
                     workspace=lq.new_workspace(1, n, k, bits), status=st2)
    torch.cuda.synchronize()
    assert int(st.item()) == LUTQ_ERR_TIMEOUT
    assert int(st2.item()) == 0
    ref_codes, ref_sb = O.quantize(w.float().numpy(), levels, bits)
    y_ref = O.gemv(x.float().numpy(), ref_codes, ref_sb, levels)
    assert O.rel_error_gate(y.cpu().numpy(), y_ref) <= 2e-3


def test_selftest_rejects_bad_arguments(lq):
    st = lq.new_status()
    with pytest.raises(lq.LutqError):
        lq.lutq_selftest_wait_timeout(st, 0)
    with pytest.raises(lq.LutqError):
        lq.lutq_selftest_wait_timeout(st, 2_000_000_000)
