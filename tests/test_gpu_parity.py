"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Codes, scales and packed bytes must match bit for bit; y must be within the
2e-3 relative gate (max |y - y_ref| / max(|y_ref|, 1e-2 * row rms)) of the fp64
oracle.  Small cases are compared in full (several tiles and a ragged split
of units across warps); the full-size workloads are compared on sampled
32-row strips, computed by the oracle on those rows alone.
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


def _cb(lq, kind, bits):
    cb = lq.lutq_codebook(kind, bits)
    ref_bits, ref_vals = O.codebook(kind, bits)
    assert np.array_equal(cb.view(torch.int16).numpy().view(np.uint16), ref_bits)
    return cb.cuda(), ref_vals


def _f32(t):
    return t.float().cpu().numpy()


def _bits16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _quantize_pack(lq, w_cpu, kind, bits):
    cb, levels = _cb(lq, kind, bits)
    st = lq.new_status()
    codes, scales = lq.lutq_quantize(w_cpu.cuda(), cb, bits, status=st)
    packed = lq.lutq_pack(codes, scales, bits, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return cb, levels, codes, scales, packed


def _gemv(lq, x_cpu, packed, scales, cb, bits, n, k, ws=None):
    m = x_cpu.shape[0]
    if ws is None:
        ws = lq.new_workspace(m, n, k, bits)
    st = lq.new_status()
    y = lq.lutq_gemv(x_cpu.cuda(), packed, cb, bits, n, k, workspace=ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return y.cpu().numpy(), ws


# ------------------------------------------------------------------ quantize

@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("logb", 4), ("lloyd_max3", 3),
                                       ("uniform4", 4)])
@pytest.mark.parametrize("n,k", [(32, 128), (96, 640), (256, 1024)])
def test_quantize_and_pack_bit_exact(lq, kind, bits, n, k):
    w = workloads.student_t_weights(n, k, 5, 0.02, seed=n + k, outlier_frac=1e-2)
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, kind, bits)
    ref_codes, ref_sb = O.quantize(_f32(w), levels, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    np.testing.assert_array_equal(_bits16(scales), ref_sb)
    np.testing.assert_array_equal(packed.cpu().numpy(), O.pack(ref_codes, ref_sb, bits))


def test_quantize_edge_cases(lq):
    # zero group, negative zeros, subnormal group, exact midpoints between levels
    kind, bits = "nf4", 4
    _, levels = O.codebook(kind, bits)
    w = np.zeros((32, 512), np.float32)
    w[1, :128] = -0.0
    m = np.random.default_rng(0).integers(-127, 128, size=128).astype(np.float64)
    w[2, 128:256] = (m * 2.0 ** -133).astype(np.float32)         # bf16 subnormals
    # midpoints: s = 1 (element 1.0 present), values at (c_i + c_{i+1}) / 2 when
    # exactly representable in bf16, else the level itself
    mids = []
    for i in range(15):
        mid = (np.float64(levels[i]) + np.float64(levels[i + 1])) / 2
        r = O.bf16_round(mid)
        mids.append(r)
    row = np.array(mids * 9, np.float32)[:127]
    w[3, 256:384] = np.concatenate([[1.0], row]).astype(np.float32)
    w[4] = O.bf16_round(np.random.default_rng(1).standard_normal(512) * 1e-30)
    wt = torch.from_numpy(w).to(torch.bfloat16)
    assert np.array_equal(wt.float().numpy(), w)
    cb, levels, codes, scales, packed = _quantize_pack(lq, wt, kind, bits)
    ref_codes, ref_sb = O.quantize(w, levels, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    np.testing.assert_array_equal(_bits16(scales), ref_sb)
    assert np.all(ref_codes[0] == 7) and np.all(ref_codes[1, :128] == 7)


def test_quantize_reports_nonfinite(lq):
    cb, _ = _cb(lq, "nf4", 4)
    w = torch.zeros((64, 256), dtype=torch.bfloat16)
    w[37, 200] = float("nan")
    st = lq.new_status()
    lq.lutq_quantize(w.cuda(), cb, 4, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5


def test_pack_reports_code_range(lq):
    codes = torch.zeros((32, 128), dtype=torch.uint8)
    codes[5, 17] = 9
    st = lq.new_status()
    scales = torch.ones((32, 1), dtype=torch.bfloat16, device="cuda")
    lq.lutq_pack(codes.cuda(), scales, 3, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 6


# ------------------------------------------------------------------ gemv

@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3), ("logb", 4)])
@pytest.mark.parametrize("m", [1, 2, 3, 8, 16])
@pytest.mark.parametrize("n,k", [(32, 128), (96, 1152), (1024, 1024), (320, 4224)])
def test_gemv_small_full_compare(lq, kind, bits, m, n, k):
    w = workloads.normal_weights(n, k, 0.02, seed=7 + n, outlier_frac=1e-3)
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, kind, bits)
    x = workloads.activations(m, k, seed=11 + m)
    y, ws = _gemv(lq, x, packed, scales, cb, bits, n, k)
    ref_codes, ref_sb = O.quantize(_f32(w), levels, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    y_ref = O.gemv(_f32(x), ref_codes, ref_sb, levels)
    assert O.rel_error_gate(y, y_ref) <= TOL
    # the workspace is left ready for the next call: a second call with it
    # gives the same bits
    y2, _ = _gemv(lq, x, packed, scales, cb, bits, n, k, ws=ws)
    np.testing.assert_array_equal(y, y2)


@pytest.mark.parametrize("bits,kind", [(4, "nf4"), (3, "lloyd_max3")])
def test_gemv_one_hot_is_exact(lq, bits, kind):
    n, k = 96, 512
    w = workloads.normal_weights(n, k, 0.02, seed=3)
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, kind, bits)
    wh = O.dequant(codes.cpu().numpy(), _bits16(scales), levels)
    ks = [0, 1, 7, 126, 127, 128, 300, 511]
    x = torch.zeros((len(ks), k), dtype=torch.bfloat16)
    for i, kk in enumerate(ks):
        x[i, kk] = 1.0
    y, _ = _gemv(lq, x, packed, scales, cb, bits, n, k)
    for i, kk in enumerate(ks):
        np.testing.assert_array_equal(y[i].astype(np.float64), wh[:, kk])


def test_gemv_deterministic_and_linear(lq):
    n, k = 4096, 4096
    w = workloads.normal_weights(n, k, 0.02, seed=5)
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, "nf4", 4)
    x = workloads.activations(1, k, seed=6)
    y1, ws = _gemv(lq, x, packed, scales, cb, 4, n, k)
    y2, _ = _gemv(lq, x, packed, scales, cb, 4, n, k, ws=ws)
    np.testing.assert_array_equal(y1, y2)
    y3, _ = _gemv(lq, (x.float() * 2).to(torch.bfloat16), packed, scales, cb, 4, n, k, ws=ws)
    np.testing.assert_array_equal(y3, 2 * y1)


# ------------------------------------------------------------------ full-size workloads

def _sample_strips(n, count=3, seed=0):
    strips = n // 32
    rng = np.random.default_rng(seed)
    pick = {0, strips - 1} | set(rng.integers(0, strips, size=count).tolist())
    return sorted(pick)


def _full_size_case(lq, lay, kind, bits, batches):
    w = lay.weights(seed=0)
    n, k = lay.n, lay.k
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, kind, bits)
    strips = _sample_strips(n)
    rows = np.concatenate([np.arange(32 * s, 32 * s + 32) for s in strips])
    w_rows = _f32(w[rows])
    ref_codes, ref_sb = O.quantize(w_rows, levels, bits)
    np.testing.assert_array_equal(codes[rows].cpu().numpy(), ref_codes)
    np.testing.assert_array_equal(_bits16(scales[rows]), ref_sb)
    # packed strips: the codes of units (s, 0..G-1) are contiguous, and so
    # are their scale blocks
    tb = 2048 if bits == 4 else 1536
    g = k // 128
    units = (n // 32) * g
    pk = packed.cpu().numpy()
    for i, s in enumerate(strips):
        want = O.pack(ref_codes[32 * i: 32 * i + 32], ref_sb[32 * i: 32 * i + 32], bits)
        np.testing.assert_array_equal(pk[s * g * tb:(s + 1) * g * tb], want[:g * tb])
        sc0 = units * tb + s * g * 64
        np.testing.assert_array_equal(pk[sc0:sc0 + g * 64], want[g * tb:])
    del w
    ws = lq.new_workspace(max(batches), n, k, bits)
    for m in batches:
        x = workloads.activations(m, k, seed=1)
        y, _ = _gemv(lq, x, packed, scales, cb, bits, n, k, ws=ws)
        y_ref = O.gemv(_f32(x), ref_codes, ref_sb, levels)
        # the gate's row rms is taken over the sampled rows of the oracle
        assert O.rel_error_gate(y[:, rows], y_ref) <= TOL, (lay.name, kind, m)


GEMV_BATCHES = (1, 2, 4, 8, 16)


@pytest.mark.parametrize("wl_name", ["tiny_w4_nf4", "w3_lm3_4096", "w4_logb_14336x4096",
                                     "llama3_8b_w4_nf4"])
def test_workload_gemv(lq, wl_name):
    wl = workloads.WORKLOADS[wl_name]
    for lay in wl.layers:
        for kind, bits in wl.codebooks:
            _full_size_case(lq, lay, kind, bits, [m for m in wl.batches if m <= 16])


@pytest.mark.parametrize("layer", ["gate_up", "down"])
@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
def test_workload_70b_gemv(lq, layer, kind, bits):
    lay = workloads.layer("llama3_70b_mlp", layer)
    _full_size_case(lq, lay, kind, bits, list(GEMV_BATCHES))


# ------------------------------------------------------------------ split strips

@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
@pytest.mark.parametrize("n,k,want_kind,want_align", [
    (1024, 8192, 1, 0),   # one helper block per strip
    (2400, 8192, 1, 0),   # two strips per helper, the last helper with one
    (5120, 8192, 0, 0),   # equal unit ranges, strips split at range ends
])
def test_gemv_split_strips(lq, kind, bits, n, k, want_kind, want_align):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = lq.lutq_gemv_plan(n, k, sms)
    if sms == 148:
        assert (plan["kind"], plan["align"]) == (want_kind, want_align), plan
    w = workloads.normal_weights(n, k, 0.02, seed=21 + n)
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, kind, bits)
    strips = list(range(n // 32)) if n * k <= (1 << 24) else _sample_strips(n, count=6)
    rows = np.concatenate([np.arange(32 * s, 32 * s + 32) for s in strips])
    ref_codes, ref_sb = O.quantize(_f32(w[rows]), levels, bits)
    np.testing.assert_array_equal(codes[rows].cpu().numpy(), ref_codes)
    ws = lq.new_workspace(3, n, k, bits)
    zero = lq.lutq_workspace_zero_bytes(3, n, k, bits)
    assert zero >= 8 * 3 * n                          # the exchange slots
    for m in (1, 3):
        x = workloads.activations(m, k, seed=31 + m)
        y, _ = _gemv(lq, x, packed, scales, cb, bits, n, k, ws=ws)
        y_ref = O.gemv(_f32(x), ref_codes, ref_sb, levels)
        assert O.rel_error_gate(y[:, rows], y_ref) <= TOL, (n, k, m)
        # the exchange slots are clear again (this shape runs on the CUDA
        # cores), and a second call gives the same bits
        assert int(ws[:zero].count_nonzero().item()) == 0
        y2, _ = _gemv(lq, x, packed, scales, cb, bits, n, k, ws=ws)
        np.testing.assert_array_equal(y, y2)


# ------------------------------------------------------------------ runs over many strips

@pytest.mark.parametrize("kind,bits", [("nf4", 4), ("lloyd_max3", 3)])
def test_gemv_warp_runs_span_strips(lq, kind, bits):
    """Two groups per row and 4096 strips: every block takes ~28 whole strips,
    so each warp's run of units crosses from strip to strip (its partial sums
    go through the block's slots at every strip end)."""
    n, k = 131072, 256
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = lq.lutq_gemv_plan(n, k, sms)
    assert plan["kind"] == 0 and plan["align"] == 1 and plan["C"] == min(sms, n // 32)
    w = workloads.normal_weights(n, k, 0.02, seed=41)
    cb, levels, codes, scales, packed = _quantize_pack(lq, w, kind, bits)
    strips = _sample_strips(n, count=8, seed=3)
    rows = np.concatenate([np.arange(32 * s, 32 * s + 32) for s in strips])
    ref_codes, ref_sb = O.quantize(_f32(w[rows]), levels, bits)
    np.testing.assert_array_equal(codes[rows].cpu().numpy(), ref_codes)
    ws = lq.new_workspace(4, n, k, bits)
    for m in (1, 2, 4):
        x = workloads.activations(m, k, seed=51 + m)
        y, _ = _gemv(lq, x, packed, scales, cb, bits, n, k, ws=ws)
        y_ref = O.gemv(_f32(x), ref_codes, ref_sb, levels)
        assert O.rel_error_gate(y[:, rows], y_ref) <= TOL, (m,)
