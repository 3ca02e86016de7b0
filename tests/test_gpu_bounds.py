"""The checked build (liblutq_bounds.so, compiled with -DLUTQ_BOUNDS) on the GPU.

The kernels of that build compare their global, shared-memory and table
indices with the buffers' extents and report LUTQ_ERR_BOUNDS through the status
word instead of making an access outside them.  Here: the self-test sees the
check fire (and, in the product build, compiled out), and the small-shape
parity tests run once against the checked build in a child process, where
every call must leave the status word at zero and every result must still
match the oracle.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUNDS_LIB = os.path.join(ROOT, "dequant_gemv_group_b200", "liblutq_bounds.so")


@pytest.fixture(scope="module")
def lq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import dequant_gemv_group_b200 as m
    return m


def test_selftest_bounds(lq):
    st = lq.new_status()
    lq.lutq_selftest_bounds(st)
    torch.cuda.synchronize()
    want = 10 if lq.lutq_build_flags() & lq.BUILD_BOUNDS else 0
    assert int(st.item()) == want


# the small-shape cases of each kernel: quantize and pack, the CUDA-core GEMV
# over its work plans, the tensor-core GEMM over its batch tiles, group 64,
# per-group types
SMALL_CASES = [
    "tests/test_gpu_parity.py::test_quantize_and_pack_bit_exact",
    "tests/test_gpu_parity.py::test_gemv_small_full_compare",
    "tests/test_gpu_parity.py::test_gemv_split_strips",
    "tests/test_gpu_parity.py::test_gemv_warp_runs_span_strips",
    "tests/test_gpu_gemm.py::test_gemm_small_full_compare",
    "tests/test_gpu_group64.py::test_quantize_and_pack_bit_exact",
    "tests/test_gpu_group64.py::test_gemv_and_gemm_against_oracle",
    "tests/test_gpu_typed.py",
    "tests/test_gpu_bounds.py::test_selftest_bounds",
]


def test_small_shapes_under_checked_build(lq):
    if os.environ.get("LUTQ_LIB_VARIANT"):
        pytest.skip("already running against a variant build")
    if not os.path.exists(BOUNDS_LIB):
        pytest.skip("liblutq_bounds.so is not built")
    env = dict(os.environ, LUTQ_LIB_VARIANT="bounds")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu",
                        "-p", "no:cacheprovider", *SMALL_CASES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-15:])
    assert r.returncode == 0, tail
    assert " passed" in tail and "failed" not in tail, tail
