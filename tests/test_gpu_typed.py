"""Per-group data types on the GPU against the oracle (through the C ABI):
codes, scales, group types and packed bytes bit for bit; the typed product
within the 2e-3 gate of the oracle's typed product, bit for bit on one-hot
activations, and bit for bit equal to lutq_gemv when every group has the
same single type."""
import numpy as np
import pytest
import torch

import workloads
from oracle import lutq_oracle as O

pytestmark = pytest.mark.gpu

TOL = 2e-3
KINDS4 = ("nf4", "logb", "uniform4")


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


def _tables(lq, bits, t):
    """Device codebooks [t, 2^bits] and the oracle's level lists."""
    if bits == 4:
        kinds = (KINDS4 + ("nf4",))[:t]
        cbs = [lq.lutq_codebook(k, 4) for k in kinds]
        levels = [O.codebook(k, 4)[1] for k in kinds]
        if t == 4:
            # a fourth type: NF4 levels shrunk by 0.75 except the two ends
            lv = O.bf16_round(levels[0].astype(np.float64) * 0.75).astype(np.float32)
            lv[0], lv[-1] = -1.0, 1.0
            levels[3] = lv
            cbs[3] = torch.from_numpy(O.bf16_bits(lv).view(np.int16)).view(torch.bfloat16)
    else:
        lm = O.codebook("lloyd_max3", 3)[1]
        levels = [lm]
        if t == 2:
            lv = O.bf16_round(lm.astype(np.float64) * 0.9).astype(np.float32)
            lv[0], lv[-1] = -1.0, 1.0
            levels.append(lv)
        cbs = [torch.from_numpy(O.bf16_bits(l).view(np.int16)).view(torch.bfloat16) for l in levels]
    return torch.stack(cbs).contiguous().cuda(), levels


_ORACLE_CACHE = {}


def _oracle_typed(w_cpu, levels, bits, key):
    """The oracle's codes, scale bits and group types of w; cached under `key`
    (a case whose weights depend only on the key) when one is given."""
    if key is None:
        return O.quantize_typed(_f32(w_cpu), levels, bits)
    if key not in _ORACLE_CACHE:
        _ORACLE_CACHE.clear()
        _ORACLE_CACHE[key] = O.quantize_typed(_f32(w_cpu), levels, bits)
    return _ORACLE_CACHE[key]


def _typed_layer(lq, w_cpu, bits, t, key=None):
    """Quantize and pack w on the GPU with t types, and check the codes,
    scales and types against the oracle's, so that every product check below
    can take the oracle's own quantization as its reference.  Returns the
    device tables, the oracle's level lists, the GPU's packed matrix and the
    oracle's (codes, scale bits, types)."""
    cbs, levels = _tables(lq, bits, t)
    st = lq.new_status()
    codes, scales, types = lq.lutq_quantize_typed(w_cpu.cuda(), cbs, bits, status=st)
    packed = lq.lutq_pack_typed(codes, scales, types, bits, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = _oracle_typed(w_cpu, levels, bits, key)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref[0])
    np.testing.assert_array_equal(_bits16(scales), ref[1])
    np.testing.assert_array_equal(types.cpu().numpy(), ref[2])
    return cbs, levels, codes, scales, types, packed, ref


CASES = [(4, 1), (4, 2), (4, 3), (4, 4), (3, 1), (3, 2)]


@pytest.mark.parametrize("bits,t", CASES)
@pytest.mark.parametrize("n,k", [(96, 1152), (1024, 4096)])
def test_quantize_and_pack_typed_bit_exact(lq, bits, t, n, k):
    w = workloads.normal_weights(n, k, 0.02, seed=n + t, outlier_frac=1e-2)
    w[5, 128:256] = 0.0                               # an all-zero group
    w[7, :128] = w[7, :128] * 2.0 ** -120             # subnormal-scaled group
    cbs, levels, codes, scales, types, packed, (rc, rs, rt) = _typed_layer(lq, w, bits, t)
    if t > 1:
        assert len(np.unique(rt)) > 1                 # the case exercises the choice
    np.testing.assert_array_equal(packed.cpu().numpy(), O.pack_typed(rc, rs, rt, bits))


@pytest.mark.parametrize("bits,t", CASES)
@pytest.mark.parametrize("m", [1, 2, 3, 4])
@pytest.mark.parametrize("n,k", [(96, 1152), (1024, 4096), (320, 4224)])
def test_gemv_typed_matches_oracle(lq, bits, t, m, n, k):
    w = workloads.normal_weights(n, k, 0.02, seed=3 * n + t, outlier_frac=1e-2)
    x = workloads.activations(m, k, seed=m + 7)
    cbs, levels, codes, scales, types, packed, (rc, rs, rt) = _typed_layer(
        lq, w, bits, t, key=("gemv", bits, t, n, k))
    st = lq.new_status()
    y = lq.lutq_gemv_typed(x.cuda(), packed, cbs, bits, n, k,
                           workspace=lq.new_workspace(m, n, k, bits), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    y_ref = O.gemv_typed(_f32(x), rc, rs, rt, levels)
    assert O.rel_error_gate(y.cpu().numpy(), y_ref) <= TOL


@pytest.mark.parametrize("bits,t", [(4, 4), (3, 2)])
def test_gemv_typed_one_hot_is_the_dequantized_weight(lq, bits, t):
    n, k = 256, 1024
    w = workloads.normal_weights(n, k, 0.02, seed=41, outlier_frac=1e-2)
    cbs, levels, codes, scales, types, packed, (rc, rs, rt) = _typed_layer(lq, w, bits, t)
    wh = O.dequant_typed(rc, rs, rt, levels)
    ws = lq.new_workspace(1, n, k, bits)
    for kk in (0, 129, 1023):
        e = torch.zeros((1, k), dtype=torch.bfloat16)
        e[0, kk] = 1.0
        y = lq.lutq_gemv_typed(e.cuda(), packed, cbs, bits, n, k, workspace=ws)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(y.cpu().numpy()[0].astype(np.float64), wh[:, kk])


@pytest.mark.parametrize("bits,kind", [(4, "nf4"), (3, "lloyd_max3")])
@pytest.mark.parametrize("m", [1, 3])
def test_single_type_equals_lutq_gemv_bitwise(lq, bits, kind, m):
    n, k = 1024, 4096
    w = workloads.normal_weights(n, k, 0.02, seed=43, outlier_frac=1e-3)
    x = workloads.activations(m, k, seed=44).cuda()
    cb = lq.lutq_codebook(kind, bits).cuda()
    codes, scales, types = lq.lutq_quantize_typed(w.cuda(), cb[None].contiguous(), bits)
    c0, s0 = lq.lutq_quantize(w.cuda(), cb, bits)
    torch.cuda.synchronize()
    assert torch.equal(codes, c0) and torch.equal(scales, s0) and not types.any()
    ws = lq.new_workspace(m, n, k, bits)
    y_t = lq.lutq_gemv_typed(x, lq.lutq_pack_typed(codes, scales, types, bits),
                             cb[None].contiguous(), bits, n, k, workspace=ws)
    y_u = lq.lutq_gemv(x, lq.lutq_pack(c0, s0, bits), cb, bits, n, k, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y_t, y_u)


def test_pack_typed_reports_out_of_range_types(lq):
    n, k = 64, 256
    codes = torch.zeros((n, k), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((n, 2), dtype=torch.bfloat16, device="cuda")
    types = torch.zeros((n, 2), dtype=torch.uint8, device="cuda")
    types[9, 1] = 2                                   # 3-bit codes allow types 0 and 1
    st = lq.new_status()
    lq.lutq_pack_typed(codes, scales, types, 3, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 6                        # LUTQ_ERR_CODE_RANGE
    st.zero_()
    lq.lutq_pack_typed(codes, scales, types, 4, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_gemv_typed_full_size_layer(lq):
    lay = workloads.layer("llama3_8b_w4_nf4", "down")
    n, k = lay.n, lay.k
    w = lay.weights(seed=0)
    cbs, levels = _tables(lq, 4, 4)
    st = lq.new_status()
    codes, scales, types = lq.lutq_quantize_typed(w.cuda(), cbs, 4, status=st)
    packed = lq.lutq_pack_typed(codes, scales, types, 4, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x = workloads.activations(1, k, seed=1)
    y = lq.lutq_gemv_typed(x.cuda(), packed, cbs, 4, n, k, workspace=lq.new_workspace(1, n, k, 4))
    torch.cuda.synchronize()
    strips = [0, 63, 127]
    rows = np.concatenate([np.arange(32 * s, 32 * s + 32) for s in strips])
    rc, rs, rt = O.quantize_typed(_f32(w[rows]), levels, 4)
    np.testing.assert_array_equal(codes[rows].cpu().numpy(), rc)
    np.testing.assert_array_equal(_bits16(scales[rows]), rs)
    np.testing.assert_array_equal(types[rows].cpu().numpy(), rt)
    y_ref = O.gemv_typed(_f32(x), rc, rs, rt, levels)
    assert O.rel_error_gate(y.cpu().numpy()[:, rows], y_ref) <= TOL
    # every type is used on this layer
    assert set(np.unique(types.cpu().numpy()).tolist()) == {0, 1, 2, 3}


@pytest.mark.parametrize("bits,t", [(4, 4), (4, 2), (3, 2)])
@pytest.mark.parametrize("m", [5, 16, 32, 64, 128])
@pytest.mark.parametrize("n,k", [(256, 1024), (320, 4224)])
def test_typed_tensor_core_path_matches_oracle(lq, bits, t, m, n, k):
    # batches beyond the CUDA-core kernel: lutq_gemv_typed (M <= 16) and
    # lutq_gemm_typed both run the tcgen05 kernel with the 128 KB table region
    w = workloads.normal_weights(n, k, 0.02, seed=5 * n + t, outlier_frac=1e-2)
    x = workloads.activations(m, k, seed=m + 11)
    cbs, levels, codes, scales, types, packed, (rc, rs, rt) = _typed_layer(
        lq, w, bits, t, key=("tc", bits, t, n, k))
    y_ref = O.gemv_typed(_f32(x), rc, rs, rt, levels)
    ws = lq.new_workspace(m, n, k, bits)
    st = lq.new_status()
    fns = [lq.lutq_gemm_typed] + ([lq.lutq_gemv_typed] if m <= 16 else [])
    for fn in fns:
        y = fn(x.cuda(), packed, cbs, bits, n, k, workspace=ws, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert O.rel_error_gate(y.cpu().numpy(), y_ref) <= TOL, fn.__name__


def test_typed_long_rows_take_the_tensor_core_path(lq):
    # M = 1 with K beyond the CUDA-core kernel's shared memory (K + 2048 > 48128)
    n, k, bits, t = 64, 128 * 380, 4, 4
    w = workloads.normal_weights(n, k, 0.02, seed=61, outlier_frac=1e-2)
    x = workloads.activations(1, k, seed=62)
    cbs, levels, codes, scales, types, packed, (rc, rs, rt) = _typed_layer(lq, w, bits, t)
    st = lq.new_status()
    y = lq.lutq_gemv_typed(x.cuda(), packed, cbs, bits, n, k,
                           workspace=lq.new_workspace(1, n, k, bits), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    y_ref = O.gemv_typed(_f32(x), rc, rs, rt, levels)
    assert O.rel_error_gate(y.cpu().numpy(), y_ref) <= TOL


@pytest.mark.parametrize("bits,t", [(4, 4), (3, 2)])
def test_typed_gemm_one_hot_is_the_dequantized_weight(lq, bits, t):
    n, k, m = 256, 1024, 32
    w = workloads.normal_weights(n, k, 0.02, seed=71, outlier_frac=1e-2)
    cbs, levels, codes, scales, types, packed, (rc, rs, rt) = _typed_layer(lq, w, bits, t)
    wh = O.dequant_typed(rc, rs, rt, levels)
    x = torch.zeros((m, k), dtype=torch.bfloat16)
    cols = (np.arange(m) * 37) % k
    x[np.arange(m), cols] = 1.0
    y = lq.lutq_gemm_typed(x.cuda(), packed, cbs, bits, n, k,
                           workspace=lq.new_workspace(m, n, k, bits))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.cpu().numpy().astype(np.float64), wh[:, cols].T)


def test_typed_gemm_single_type_equals_lutq_gemm_bitwise(lq):
    n, k, m, bits = 512, 2048, 64, 4
    w = workloads.normal_weights(n, k, 0.02, seed=73, outlier_frac=1e-3)
    x = workloads.activations(m, k, seed=74).cuda()
    cb = lq.lutq_codebook("nf4", bits).cuda()
    codes, scales, types = lq.lutq_quantize_typed(w.cuda(), cb[None].contiguous(), bits)
    ws = lq.new_workspace(m, n, k, bits)
    y_t = lq.lutq_gemm_typed(x, lq.lutq_pack_typed(codes, scales, types, bits),
                             cb[None].contiguous(), bits, n, k, workspace=ws)
    y_u = lq.lutq_gemm(x, lq.lutq_pack(codes, scales, bits), cb, bits, n, k, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y_t, y_u)


@pytest.mark.parametrize("t", [2, 4])
def test_typed_route_by_table_region(lq, t):
    # M = 4, K = 14336: 4 * (K + 2048) = 65536 fits the CUDA-core kernel with
    # 64 KB of tables (two 4-bit types) but not with 128 KB (four), which
    # then runs on the tensor cores; both within the gate
    n, k, m, bits = 256, 14336, 4, 4
    w = workloads.normal_weights(n, k, 0.02, seed=81 + t, outlier_frac=1e-2)
    x = workloads.activations(m, k, seed=82)
    cbs, levels, codes, scales, types, packed, (rc, rs, rt) = _typed_layer(lq, w, bits, t)
    st = lq.new_status()
    y = lq.lutq_gemv_typed(x.cuda(), packed, cbs, bits, n, k,
                           workspace=lq.new_workspace(m, n, k, bits), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    y_ref = O.gemv_typed(_f32(x), rc, rs, rt, levels)
    assert O.rel_error_gate(y.cpu().numpy(), y_ref) <= TOL


@pytest.mark.parametrize("bits,t_data,t_call,m", [(4, 4, 1, 1), (4, 4, 2, 2), (4, 4, 2, 32),
                                                  (3, 2, 1, 1), (3, 2, 1, 32)])
def test_types_beyond_the_count_stay_inside_the_tables(lq, bits, t_data, t_call, m):
    # a matrix quantized with more types than the call passes: the lookups of
    # the extra types are masked to the smaller table region (values
    # unspecified, every access in bounds), the call reports
    # LUTQ_ERR_CODE_RANGE, and the call and the device stay sound
    n, k = 256, 2048
    w = workloads.normal_weights(n, k, 0.02, seed=91, outlier_frac=1e-2)
    x = workloads.activations(m, k, seed=92).cuda()
    cbs, levels, codes, scales, types, packed, (rc, rs, rt) = _typed_layer(lq, w, bits, t_data)
    assert int(types.max().item()) >= t_call
    fn = lq.lutq_gemv_typed if m <= 16 else lq.lutq_gemm_typed
    st = lq.new_status()
    fn(x, packed, cbs[:t_call].contiguous(), bits, n, k,
       workspace=lq.new_workspace(m, n, k, bits), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 6                        # LUTQ_ERR_CODE_RANGE
    # the correct call afterwards is still exact
    y = fn(x, packed, cbs, bits, n, k, workspace=lq.new_workspace(m, n, k, bits))
    torch.cuda.synchronize()
    y_ref = O.gemv_typed(_f32(x.cpu()), rc, rs, rt, levels)
    assert O.rel_error_gate(y.cpu().numpy(), y_ref) <= TOL
