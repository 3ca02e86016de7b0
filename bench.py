"""Benchmark of the fused LUT-dequant GEMV (and the tensor-core GEMM) on B200.

One step = one product call y = x * dequant(W)^T on one synthetic batch, the
hot path of inference; quantization and packing are offline (once per layer)
and run before the timed region.  Default workload: the Llama-3-8B-shaped
down projection W[4096, 14336], 4-bit NormalFloat, group 128, batch 1.

Timing: W warm-up steps, then exactly K steps between a barrier and
torch.cuda.synchronize() on both sides, CUDA events on the launching stream,
max over ranks.  The K launches are replayed from CUDA graphs, queued behind a
short spin kernel that ends before the start event, so the host's launch
latency is not in the timed region.  The weights
rotate over R device copies whose total exceeds 3x the L2 size, so no step
finds its weights in L2.  `e2e` times the same steps through the public call
with x copied from pinned host memory and y read back every step.

`--impl reference` times the CPU oracle (test infrastructure) on the same
workload, on a bounded sample of rows per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100000)
    p.add_argument("--warmup", type=int, default=2000)
    p.add_argument("--impl", default="lutq", choices=["lutq", "reference"])
    p.add_argument("--workload", default="llama3_8b_w4_nf4")
    p.add_argument("--layer", default="down")
    p.add_argument("--codebook", default="nf4")
    p.add_argument("--bits", type=int, default=4)
    p.add_argument("--batch", type=int, default=1)
    p.add_argument("--e2e-steps", type=int, default=5000)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-side", action="store_true", help="skip the GEMM and offline lines")
    p.add_argument("--table", action="store_true",
                   help="instead of the JSON line: every workload x layer x codebook x batch, "
                        "plus batches 17-31 and one scale per group of 64, as a markdown table")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def algorithmic_bytes(m, n, k, bits):
    packed = n * k // 2 if bits == 4 else 3 * n * k // 8
    return packed + n * (k // 128) * 2 + m * k * 2 + m * n * 4


GEMV_SOURCES = ("lutq_common.cuh", "lutq_lut.cuh", "lutq_gemv.cu")
GEMM_SOURCES = ("lutq_common.cuh", "lutq_lut.cuh", "lutq_sm100.cuh", "lutq_gemm.cu")


def kernel_source_sha(files):
    src = os.path.join(ROOT, "dequant_gemv_group_b200", "csrc")
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(src, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, files):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(kernel_key)
    if not d or d.get("source_sha") != kernel_source_sha(files):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clocks and clock-event reasons of one GPU, read through NVML by a
    thread every 0.5 ms from start() to stop(), plus explicit reads at the
    edges of the timed region (mark()), so that even a timed region shorter
    than the polling interval has samples taken while the GPU was busy."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device):
        import threading
        self.samples, self.marks, self.reasons = [], [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.handle = None
        try:
            import pynvml
            self.nv = pynvml
            pynvml.nvmlInit()
            uuid = str(getattr(torch.cuda.get_device_properties(device), "uuid", ""))
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(int(device))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle,
                                                                  pynvml.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: report why
            self.error = f"nvml unavailable: {e}"

    def _read(self):
        nv = self.nv
        mhz = float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        for name, const in self.REASONS:
            if bits & getattr(nv, const, 0):
                self.reasons.add(name)
        return mhz

    def _poll(self):
        import time as _t
        while not self._stop.is_set():
            try:
                self.samples.append(self._read())
            except Exception:
                pass
            _t.sleep(0.0005)

    def start(self):
        import threading
        if self.handle is None:
            return
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()

    def mark(self):
        if self.handle is not None:
            try:
                self.marks.append(self._read())
            except Exception:
                pass

    def stop(self):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [getattr(self, "error", "")],
                    "samples": 0}
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        allv = self.samples + self.marks
        busy = [v for v in allv if self.max_mhz and v >= 0.5 * self.max_mhz] or allv
        return {"sm_mhz": float(np.median(busy)) if busy else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(allv),
                "edge_mhz": self.marks, "source": "nvml, 0.5 ms polling + reads at the "
                                                  "timed region's edges"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(world, value):
    """The largest of the ranks' values (a time: the job takes as long as its
    slowest rank).  NCCL reduces on the device, other backends on the host."""
    if world == 1:
        return value
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(bytes_per_step, steps, max_seconds, world):
    """Whole-job GB/s: the bytes all ranks processed (each rank runs the same
    steps on its own replica) over the slowest rank's time."""
    return bytes_per_step * steps * world / max_seconds / 1e9


# ---------------------------------------------------------------------- oracle arm

def oracle_sample(lay, kind, bits, m, rows):
    from oracle import lutq_oracle as O
    w = lay.weights(seed=0)[:rows].float().numpy()
    _, levels = O.codebook(kind, bits)
    codes, sb = O.quantize(w, levels, bits)
    x = workloads.activations(m, lay.k, seed=1).float().numpy()
    return O, x, codes, sb, levels


def oracle_threads():
    """Threads the oracle's BLAS pool uses (all the cores this process may run on)."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def limited_threads(n):
    """A context in which the oracle's BLAS pool uses n threads."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=n, user_api="blas")
    except Exception:
        import contextlib
        return contextlib.nullcontext()


def time_oracle(lay, kind, bits, m, rows, seconds=None, calls=None):
    O, x, codes, sb, levels = oracle_sample(lay, kind, bits, m, rows)
    O.gemv(x, codes, sb, levels)
    n_calls, t0 = 0, time.perf_counter()
    while True:
        O.gemv(x, codes, sb, levels)
        n_calls += 1
        el = time.perf_counter() - t0
        if (calls is not None and n_calls >= calls) or (seconds is not None and el >= seconds):
            break
    per_call = el / n_calls
    gbs = algorithmic_bytes(m, rows, lay.k, bits) / per_call / 1e9
    return gbs, per_call, n_calls


def run_reference(args, world, rank):
    if rank != 0:
        return
    lay = workloads.layer(args.workload, args.layer)
    m = args.batch
    # rows per step sized so that warm-up + timed steps take about a minute:
    # the cost of one row is calibrated on a 64-row sample first
    _, per_call, _ = time_oracle(lay, args.codebook, args.bits, m, 64, calls=3)
    per_step = 60.0 / max(1, args.steps + args.warmup)
    rows = max(1, min(lay.n, int(per_step / (per_call / 64))))
    O, x, codes, sb, levels = oracle_sample(lay, args.codebook, args.bits, m, rows)
    for _ in range(args.warmup):
        O.gemv(x, codes, sb, levels)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.gemv(x, codes, sb, levels)
    el = time.perf_counter() - t0
    gbs = algorithmic_bytes(m, rows, lay.k, args.bits) * args.steps / el / 1e9
    sample = f"{rows} of {lay.n} rows of the layer per step (oracle-quantized), fp64 numpy"
    cores = oracle_threads()  # the BLAS pool spans the process's cores
    line = {
        "impl": "reference", "metric": "dequant-fused GEMV HBM GB/s", "value": gbs,
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args, lay),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "cpu": cpu_model(),
                         "affinity_cores": len(os.sched_getaffinity(0))},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(args, lay):
    return {"workload": f"{args.workload}/{lay.name} W[{lay.n},{lay.k}] {args.codebook} "
                        f"W{args.bits} group128 batch{args.batch}",
            "N": lay.n, "K": lay.k, "M": args.batch, "bits": args.bits,
            "codebook": args.codebook, "group": 128}


# ---------------------------------------------------------------------- lutq arm

def capture(fn, count):
    """A CUDA graph of fn(0) .. fn(count - 1), uploaded to the device, so that
    its first replay does not also pay for moving the graph there."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(count):
            fn(i)
    try:
        from cuda.bindings import driver as cu
        err, = cu.cuGraphUpload(cu.CUgraphExec(g.raw_cuda_graph_exec()),
                                cu.CUstream(torch.cuda.current_stream().cuda_stream))
        if err != cu.CUresult.CUDA_SUCCESS:
            raise RuntimeError(str(err))
        torch.cuda.synchronize()
    except Exception as e:  # the graph still replays; its first replay uploads it
        print(f"bench: graph upload skipped ({e})", file=sys.stderr)
    return g


def hold_stream(cycles=200_000):
    """Keep the current stream busy for `cycles` SM clocks (about 100 us) with
    a spin kernel, so that the launches queued after it (and the start event
    before them) are already on the device when it ends: the event pair then
    times the device work alone, not the host's launch latency (the
    blocking-kernel method of NVIDIA's nvbench).  The spin runs before the
    start event."""
    torch.cuda._sleep(int(cycles))


def time_graph(fn, count, replays=5):
    """Median device time per call of fn(0) .. fn(count - 1) replayed from an
    uploaded CUDA graph behind the stream-holding spin (after 3 warm-up calls)."""
    for i in range(3):
        fn(i)
    g = capture(fn, count)
    g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(replays):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hold_stream()
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) / 1e3 / count)
    del g
    return float(np.median(ts))


def time_events(fn, reps):
    """Average device time of fn() over reps calls (CUDA events, current stream)."""
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(reps):
        fn(i)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / reps


def side_measurements(lq, dev, args):
    """The rest of the metric and the offline steps, each on its own workload:
    the tensor-core GEMM at batch 128 on the 70B-shaped gate/up layer (TFLOP/s
    against the measured bf16 peak) and quantize + pack of the headline layer."""
    out = {}
    hbm_peak, tf_peak, peak_kind = peaks()
    lay = workloads.layer("llama3_70b_mlp", "gate_up")
    n, k, bits, m = lay.n, lay.k, 4, 128
    cb = lq.lutq_codebook("nf4", bits).to(dev)
    w = lay.weights(seed=0).to(dev)
    st = lq.new_status(dev)
    codes, scales = lq.lutq_quantize(w, cb, bits, status=st)
    packed = lq.lutq_pack(codes, scales, bits, status=st)
    del w, codes, scales
    x = workloads.activations(m, k, seed=1).to(dev)
    y = torch.empty((m, n), dtype=torch.float32, device=dev)
    ws = lq.new_workspace(m, n, k, bits, dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(2, int(np.ceil(3 * l2 / packed.numel())) + 1)
    packs_g = [packed] + [packed.clone() for _ in range(copies - 1)]
    call = lambda i: lq.lutq_gemm(x, packs_g[i % copies], cb, bits, n, k, y=y, workspace=ws,
                                  status=st)
    s = time_graph(call, 20)
    assert int(st.item()) == 0
    tflops = 2.0 * m * n * k / s / 1e12
    nbytes = packed.numel() + m * k * 2 + m * n * 4
    out["gemm"] = {"workload": f"llama3_70b_mlp/gate_up W[{n},{k}] nf4 W4 group128 batch{m}",
                   "metric": "GEMM TFLOP/s at batch>=32", "value": tflops, "unit": "TFLOP/s",
                   "us": s * 1e6, "hbm_gbs": nbytes / s / 1e9,
                   "roofline": {"bound": "tensor", "achieved": tflops, "peak": tf_peak,
                                "unit": "TFLOP/s", "frac": tflops / tf_peak,
                                "peak_source": peak_kind + " (bf16 burst)",
                                "traffic": ncu_traffic(f"gemm_w4_m{m}_{n}x{k}", GEMM_SOURCES)},
                   "kernel": "lutq::gemm_kernel"}
    del packed, packs_g, x, y, ws
    # offline steps on the headline layer
    lay = workloads.layer(args.workload, args.layer)
    n, k, bits = lay.n, lay.k, args.bits
    cb = lq.lutq_codebook(args.codebook, bits).to(dev)
    w = lay.weights(seed=0).to(dev)
    codes, scales = lq.lutq_quantize(w, cb, bits, status=st)
    tq = time_events(lambda i: lq.lutq_quantize(w, cb, bits, status=st), 10)
    tp = time_events(lambda i: lq.lutq_pack(codes, scales, bits, status=st), 10)
    assert int(st.item()) == 0
    q_bytes = n * k * 2 + n * k + n * (k // 128) * 2
    p_bytes = n * k + (n * k * bits) // 8 + 2 * n * (k // 128) * 2
    # randomized Hadamard rotation fused into the GEMV, batch 1, on the same
    # layer: throughput (graph-replayed, weights rotating over copies larger
    # than L2) and the product's error against the unquantized one with and
    # without the rotation
    signs = workloads.rht_signs(1).to(dev)
    x1 = workloads.activations(1, k, seed=1).to(dev)
    y1 = torch.empty((1, n), dtype=torch.float32, device=dev)
    ws1 = lq.new_workspace(1, n, k, bits, dev)
    packed_plain = lq.lutq_pack(codes, scales, bits, status=st)
    wr = lq.lutq_rht_weights(w, signs)
    codes_r, scales_r = lq.lutq_quantize(wr, cb, bits, status=st)
    packed_r = lq.lutq_pack(codes_r, scales_r, bits, status=st)
    del wr, codes_r, scales_r
    copies = max(2, int(np.ceil(3 * l2 / packed_r.numel())) + 1)
    packs_r = [packed_r] + [packed_r.clone() for _ in range(copies - 1)]
    call_r = lambda i: lq.lutq_gemv_rht(x1, packs_r[i % copies], cb, signs, bits, n, k, y=y1,
                                        workspace=ws1, status=st)
    for i in range(4):
        call_r(i)
    g_r = capture(call_r, 128)
    g_r.replay()
    t_r = time_events(lambda i: g_r.replay(), 8) / 128
    del g_r
    exact = (x1.double() @ w.double().t()).cpu().numpy()
    y_plain = lq.lutq_gemv(x1, packed_plain, cb, bits, n, k, workspace=ws1, status=st)
    y_rot = lq.lutq_gemv_rht(x1, packed_r, cb, signs, bits, n, k, workspace=ws1, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    err_plain = float(np.linalg.norm(y_plain.double().cpu().numpy() - exact) / np.linalg.norm(exact))
    err_rot = float(np.linalg.norm(y_rot.double().cpu().numpy() - exact) / np.linalg.norm(exact))
    out["rht"] = {"workload": f"{args.workload}/{args.layer} W[{n},{k}] {args.codebook} W{bits} "
                              "batch1, activations rotated in the GEMV prologue",
                  "value": algorithmic_bytes(1, n, k, bits) / t_r / 1e9, "unit": "GB/s",
                  "us": t_r * 1e6, "kernel": "lutq::gemv_small_kernel (rotating)",
                  "rel_error_vs_unquantized": {"plain": err_plain, "rotated": err_rot}}
    del packs_r, packed_r, packed_plain
    # codebook fitted to the same layer: the histogram pass (GB/s of weights
    # read) and the product's error against the unquantized one, starting
    # codebook against fitted
    hist = torch.zeros(lq.HIST_BINS, dtype=torch.int64, device=dev)
    lq.lutq_fit_histogram(w, hist=hist, status=st)
    th = time_events(lambda i: lq.lutq_fit_histogram(w, hist=hist, status=st), 5)
    hist.zero_()
    lq.lutq_fit_histogram(w, hist=hist, status=st)
    fitted = lq.lutq_fit_codebook(hist.cpu(), bits, cb.cpu()).to(dev)
    codes_f, scales_f = lq.lutq_quantize(w, fitted, bits, status=st)
    y_fit = lq.lutq_gemv(x1, lq.lutq_pack(codes_f, scales_f, bits, status=st), fitted, bits, n, k,
                         workspace=ws1, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    err_fit = float(np.linalg.norm(y_fit.double().cpu().numpy() - exact) / np.linalg.norm(exact))
    out["fitted_codebook"] = {"histogram_gbs": n * k * 2 / th / 1e9, "histogram_us": th * 1e6,
                              "rel_error_vs_unquantized": {args.codebook: err_plain,
                                                           "fitted": err_fit},
                              "note": "Lloyd-Max on the layer's normalised weights from "
                                      f"{args.codebook}; same GEMV"}
    del codes_f, scales_f
    # per-group data types on the same layer: the codebooks of the run, then
    # (4-bit) log-b and uniform, and the fitted one; each group takes the type
    # of smallest error.  Throughput of the typed GEMV at batch 1 (graph
    # replay, weights rotating over copies larger than L2), the typed
    # quantizer's time, and the product's error against the unquantized one
    tables = [cb] + ([lq.lutq_codebook("logb", 4).to(dev), lq.lutq_codebook("uniform4", 4).to(dev)]
                     if bits == 4 else []) + [fitted]
    tables = tables[:lq.lutq_max_types(bits)]
    cbs = torch.stack(tables).contiguous()
    codes_t, scales_t, types_t = lq.lutq_quantize_typed(w, cbs, bits, status=st)
    tt = time_events(lambda i: lq.lutq_quantize_typed(w, cbs, bits, status=st), 1)
    packed_t = lq.lutq_pack_typed(codes_t, scales_t, types_t, bits, status=st)
    counts = torch.bincount(types_t.reshape(-1).long(), minlength=len(tables)).cpu().tolist()
    del codes_t, scales_t, types_t
    copies = max(2, int(np.ceil(3 * l2 / packed_t.numel())) + 1)
    packs_t = [packed_t] + [packed_t.clone() for _ in range(copies - 1)]
    call_t = lambda i: lq.lutq_gemv_typed(x1, packs_t[i % copies], cbs, bits, n, k, y=y1,
                                          workspace=ws1, status=st)
    for i in range(4):
        call_t(i)
    g_t = capture(call_t, 128)
    g_t.replay()
    t_t = time_events(lambda i: g_t.replay(), 8) / 128
    del g_t
    y_typed = lq.lutq_gemv_typed(x1, packed_t, cbs, bits, n, k, workspace=ws1, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    err_typed = float(np.linalg.norm(y_typed.double().cpu().numpy() - exact) / np.linalg.norm(exact))
    typed_bytes = algorithmic_bytes(1, n, k, bits) + (n // 32) * (k // 128) * 8
    out["typed"] = {"workload": f"{args.workload}/{args.layer} W[{n},{k}] W{bits} batch1, "
                                f"{len(tables)} codebooks chosen per group of 128",
                    "value": typed_bytes / t_t / 1e9, "unit": "GB/s", "us": t_t * 1e6,
                    "kernel": "lutq::gemv_small_kernel (typed)",
                    "quantize_typed_us": tt * 1e6, "groups_per_type": counts,
                    "rel_error_vs_unquantized": {args.codebook: err_plain, "typed": err_typed}}
    del packs_t, packed_t
    # one scale per group of 64 on the same layer: the GEMV at batch 1
    # (graph replay, weights rotating over copies larger than L2), the
    # tensor-core GEMM at batch 128, and the product's error against the
    # unquantized one
    codes_h, scales_h = lq.lutq_quantize_group64(w, cb, bits, status=st)
    packed_h = lq.lutq_pack_group64(codes_h, scales_h, bits, status=st)
    del codes_h, scales_h
    copies = max(2, int(np.ceil(3 * l2 / packed_h.numel())) + 1)
    packs_h = [packed_h] + [packed_h.clone() for _ in range(copies - 1)]
    call_h = lambda i: lq.lutq_gemv_group64(x1, packs_h[i % copies], cb, bits, n, k, y=y1,
                                            workspace=ws1, status=st)
    for i in range(4):
        call_h(i)
    g_h = capture(call_h, 128)
    g_h.replay()
    t_h = time_events(lambda i: g_h.replay(), 8) / 128
    del g_h
    y_h = lq.lutq_gemv_group64(x1, packed_h, cb, bits, n, k, workspace=ws1, status=st)
    mg = 128
    xg = workloads.activations(mg, k, seed=1).to(dev)
    yg = torch.empty((mg, n), dtype=torch.float32, device=dev)
    wsg = lq.new_workspace(mg, n, k, bits, dev)
    call_g = lambda i: lq.lutq_gemm_group64(xg, packs_h[i % copies], cb, bits, n, k, y=yg,
                                            workspace=wsg, status=st)
    t_g = time_graph(call_g, 20)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    err_h = float(np.linalg.norm(y_h.double().cpu().numpy() - exact) / np.linalg.norm(exact))
    h_bytes = algorithmic_bytes(1, n, k, bits) + n * (k // 128) * 2   # two scales per 128
    out["group64"] = {"workload": f"{args.workload}/{args.layer} W[{n},{k}] {args.codebook} "
                                  f"W{bits} group64 batch1",
                      "value": h_bytes / t_h / 1e9, "unit": "GB/s", "us": t_h * 1e6,
                      "frac_of_hbm_peak": h_bytes / t_h / 1e9 / hbm_peak,
                      "kernel": "lutq::gemv_small_kernel (128-byte scale blocks)",
                      "gemm_batch128": {"us": t_g * 1e6,
                                        "tflops": 2.0 * mg * n * k / t_g / 1e12,
                                        "kernel": "lutq::gemm_kernel (two partials per unit)"},
                      "rel_error_vs_unquantized": {f"{args.codebook}_group128": err_plain,
                                                   f"{args.codebook}_group64": err_h}}
    del packs_h, packed_h, xg, yg, wsg
    # the baselines of the pages' quantizers, same layer, same GEMV: one scale
    # per row, and the tensor-wise asymmetric linear quantizer (levels evenly
    # spaced from min W to max W, one scale for the matrix)
    errs = {}
    codes_b, scales_b = lq.lutq_quantize_rowscale(w, cb, bits, status=st)
    y_b = lq.lutq_gemv(x1, lq.lutq_pack(codes_b, scales_b, bits, status=st), cb, bits, n, k,
                       workspace=ws1, status=st)
    errs[f"{args.codebook}_row_scale"] = y_b
    wmin, wmax = float(w.float().min()), float(w.float().max())
    cb_a = lq.lutq_codebook_asym_linear(wmin, wmax, bits).to(dev)
    codes_b, scales_b = lq.lutq_quantize_tensorscale(w, cb_a, bits, status=st)
    y_b = lq.lutq_gemv(x1, lq.lutq_pack(codes_b, scales_b, bits, status=st), cb_a, bits, n, k,
                       workspace=ws1, status=st)
    errs["asym_linear_tensor_scale"] = y_b
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    out["baselines"] = {"rel_error_vs_unquantized": dict(
        {f"{args.codebook}_group128": err_plain},
        **{key: float(np.linalg.norm(v.double().cpu().numpy() - exact) / np.linalg.norm(exact))
           for key, v in errs.items()}),
        "note": "same layer and GEMV; scales per group of 128, per row, or one per matrix"}
    del codes_b, scales_b, errs
    out["offline"] = {"quantize_gbs": q_bytes / tq / 1e9, "quantize_us": tq * 1e6,
                      "pack_gbs": p_bytes / tp / 1e9, "pack_us": tp * 1e6,
                      "note": "W bf16 -> codes u8 + scales; codes + scales -> layout V2 (L2-warm)"}
    return out


# batches between the GEMV's 16 and 32 on the 70B-shaped layers, and the
# group-64 cases of the per-configuration table
TABLE_EXTRA_BATCHES = {"llama3_70b_mlp": (17, 20, 24, 28, 31)}
TABLE_GROUP64 = {("llama3_8b_w4_nf4", "down"): (1, 4, 16, 32, 128),
                 ("llama3_70b_mlp", "gate_up"): (1, 4, 16, 32, 128)}


def run_table(args):
    """Per-configuration table: each product graph-replayed (9 replays of 64
    calls behind a spin kernel, weights rotating over copies larger than 3x
    L2); median (p10-p90) microseconds per call, GB/s of algorithmic bytes,
    percent of 8 TB/s and TFLOP/s, one markdown row each."""
    import dequant_gemv_group_b200 as lq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    print("| config | layer | W[N,K] | codebook | group | M | call | us median (p10-p90) "
          "| GB/s | % of 8 TB/s | TFLOP/s |")
    print("|---|---|---|---|---|---|---|---|---|---|---|")

    def sweep(wname, lay, kind, bits, group, batches, packed, cb):
        n, k = lay.n, lay.k
        per = packed.numel()
        copies = max(2, int(np.ceil(3 * l2 / per)) + 1)
        packs = [packed] + [packed.clone() for _ in range(copies - 1)]
        st = lq.new_status(dev)
        for m in batches:
            if group == 64:
                fn = lq.lutq_gemv_group64 if m <= 16 else lq.lutq_gemm_group64
            else:
                fn = lq.lutq_gemv if m <= 16 else lq.lutq_gemm
            x = workloads.activations(m, k, seed=1).to(dev)
            y = torch.empty((m, n), device=dev)
            ws = lq.new_workspace(m, n, k, bits, dev)
            step = lambda i: fn(x, packs[i % copies], cb, bits, n, k, y=y, workspace=ws,
                                status=st)
            for i in range(5):
                step(i)
            g = capture(step, 64)
            g.replay()
            torch.cuda.synchronize()
            ts = []
            for _ in range(9):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                hold_stream()
                e0.record()
                g.replay()
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3 / 64)
            assert int(st.item()) == 0, (wname, lay.name, m)
            med, p10, p90 = np.median(ts), np.percentile(ts, 10), np.percentile(ts, 90)
            gbs = (per + m * k * 2 + m * n * 4) / med / 1e3
            tf = 2.0 * m * n * k / med / 1e6
            print(f"| {wname} | {lay.name} | {n}x{k} | {kind} W{bits} | {group} | {m} | "
                  f"{fn.__name__} | {med:.2f} ({p10:.2f}-{p90:.2f}) | {gbs:.0f} | "
                  f"{gbs / 80:.1f} | {tf:.1f} |", flush=True)
            del g, x, y, ws
        del packs

    for wname, wl in workloads.WORKLOADS.items():
        for lay in wl.layers:
            w = lay.weights(seed=0).to(dev)
            for kind, bits in wl.codebooks:
                cb = lq.lutq_codebook(kind, bits).to(dev)
                codes, scales = lq.lutq_quantize(w, cb, bits)
                packed = lq.lutq_pack(codes, scales, bits)
                del codes, scales
                batches = tuple(sorted(set(wl.batches) | set(TABLE_EXTRA_BATCHES.get(wname, ()))))
                sweep(wname, lay, kind, bits, 128, batches, packed, cb)
                del packed
                g64 = TABLE_GROUP64.get((wname, lay.name))
                if g64 and bits == 4:
                    codes, scales = lq.lutq_quantize_group64(w, cb, bits)
                    packed = lq.lutq_pack_group64(codes, scales, bits)
                    del codes, scales
                    sweep(wname, lay, kind, bits, 64, g64, packed, cb)
                    del packed
            del w
            torch.cuda.empty_cache()


def run_lutq(args, world, rank, local):
    import dequant_gemv_group_b200 as lq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lay = workloads.layer(args.workload, args.layer)
    n, k, m, bits = lay.n, lay.k, args.batch, args.bits

    cb = lq.lutq_codebook(args.codebook, bits).to(dev)
    w = lay.weights(seed=0).to(dev)
    st = lq.new_status(dev)
    codes, scales = lq.lutq_quantize(w, cb, bits, status=st)
    packed = lq.lutq_pack(codes, scales, bits, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    del w, codes, scales

    per_copy = packed.numel()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(2, int(np.ceil(3 * l2 / per_copy)) + 1)
    packs = [packed] + [packed.clone() for _ in range(copies - 1)]
    x = workloads.activations(m, k, seed=1).to(dev)
    y = torch.empty((m, n), dtype=torch.float32, device=dev)
    ws = lq.new_workspace(m, n, k, bits, dev)
    use_gemm = m > 16
    call = lq.lutq_gemm if use_gemm else lq.lutq_gemv
    # the kernel that runs the step: lutq_gemv keeps batches of up to 4 on the
    # CUDA cores when M (K + 2048) <= 80896 (the activations fit its shared
    # memory, include/lutq.h) and hands the others to the tensor-core kernel
    cuda_core = (not use_gemm) and m <= 4 and m * (k + 2048) <= 80896

    def step(i):
        j = i % copies
        call(x, packs[j], cb, bits, n, k, y=y, workspace=ws, status=st)

    for i in range(8):  # eager warm-up (module load, attributes)
        step(i)
    torch.cuda.synchronize()

    chunk = min(512, max(1, args.steps))
    g_chunk = capture(step, chunk)
    rem = args.steps % chunk
    g_rem = capture(step, rem) if rem else None
    w_graph = capture(step, args.warmup) if 0 < args.warmup <= 4096 else None

    stream = torch.cuda.current_stream()
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    if w_graph is not None:
        w_graph.replay()
    else:
        for i in range(args.warmup):
            step(i)
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hold_stream()
    ev0.record(stream)
    for _ in range(args.steps // chunk):
        g_chunk.replay()
    if g_rem is not None:
        g_rem.replay()
    ev1.record(stream)
    sampler.mark()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(world, ms)
    assert int(st.item()) == 0
    if clocks.get("sm_mhz"):
        clocks["sm_cycles_per_step"] = ms / args.steps * 1e-3 * clocks["sm_mhz"] * 1e6

    # context for the timed number: one call on an idle GPU (nothing to
    # overlap its start with), and the per-call time of long graph replays
    # (steady state: every call's start overlaps the previous call's end)
    iso = []
    for i in range(20):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hold_stream()
        e0.record(stream)
        step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        iso.append(e0.elapsed_time(e1) * 1e3)
    reps = max(1, min(16, 4096 // chunk))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g_chunk.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    steady_us = e0.elapsed_time(e1) * 1e3 / (reps * chunk)

    nbytes = algorithmic_bytes(m, n, k, bits)
    per_step_s = ms / 1e3 / args.steps
    gbs_rank = nbytes / per_step_s / 1e9          # one GPU (the slowest rank)
    value = aggregate_rate(nbytes, args.steps, ms / 1e3, world)

    # plain stream launches (no graph), for context
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    plain_steps = min(args.steps, 20000)
    e0.record(stream)
    for i in range(plain_steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    plain_gbs = nbytes / (e0.elapsed_time(e1) / 1e3 / plain_steps) / 1e9

    # end to end through the public call with host buffers
    x_host = workloads.activations(m, k, seed=1).pin_memory()
    y_host = torch.empty((m, n), dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(x)
    e2e_steps = min(args.steps, args.e2e_steps)
    for i in range(20):
        x_dev.copy_(x_host, non_blocking=True)
        call(x_dev, packs[i % copies], cb, bits, n, k, y=y, workspace=ws)
        y_host.copy_(y, non_blocking=True)
        torch.cuda.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    for i in range(e2e_steps):
        x_dev.copy_(x_host, non_blocking=True)
        call(x_dev, packs[i % copies], cb, bits, n, k, y=y, workspace=ws)
        y_host.copy_(y, non_blocking=True)
        torch.cuda.synchronize()
    e2e_s = max_over_ranks(world, time.perf_counter() - t0)
    e2e_gbs = aggregate_rate(nbytes, e2e_steps, e2e_s, world)

    extra = side_measurements(lq, dev, args) if not args.no_side else {}

    hbm_peak, tf_peak, peak_kind = peaks()
    kernel_key = f"gemv_w{bits}_m{m}_{n}x{k}"
    line = {
        "metric": "dequant-fused GEMV HBM GB/s", "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(args, lay),
        "timing": {"parallelism": f"replicas{world}", "launch": "cuda_graph",
                   "l2": f"weights rotate over {copies} copies "
                         f"({copies * per_copy / 1e6:.0f} MB > 3x L2 {l2 / 1e6:.0f} MB); "
                         "graphs uploaded to the device before the timed region",
                   "isolated_call_us": float(np.median(iso)),
                   "steady_state_us": steady_us,
                   "steady_state_gbs": nbytes / steady_us / 1e3},
        "roofline": {"bound": "hbm", "achieved": gbs_rank, "peak": hbm_peak, "unit": "GB/s",
                     "frac": gbs_rank / hbm_peak, "peak_source": peak_kind,
                     "bytes_per_launch": nbytes,
                     "traffic": ncu_traffic(kernel_key, GEMV_SOURCES if cuda_core else GEMM_SOURCES),
                     "kernel": "lutq::gemv_small_kernel" if cuda_core else "lutq::gemm_kernel"},
        "pct_of_8TBs": gbs_rank / 8000.0,
        "plain_launch_gbs": plain_gbs,
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": m * k * 2,
                "d2h_bytes_per_step": m * n * 4, "steps": e2e_steps,
                "note": "x H2D + product + y D2H + host sync per step"},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    line.update(extra)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        rows = 512
        with limited_threads(1):
            gbs_1, per_call_1, calls_1 = time_oracle(lay, args.codebook, bits, m, rows,
                                                     seconds=8.0)
        gbs_cpu, per_call, calls = time_oracle(lay, args.codebook, bits, m, rows, seconds=8.0)
        line["cpu_baseline"] = {
            "value": gbs_cpu, "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{rows} of {n} rows (oracle-quantized), {calls} calls of the oracle "
                      f"product, {per_call * 1e3:.1f} ms each",
            "single_thread": {"value": gbs_1, "unit": "GB/s", "calls": calls_1,
                              "ms_per_call": per_call_1 * 1e3},
            "cpu": cpu_model(), "affinity_cores": len(os.sched_getaffinity(0))}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.table:
        run_table(args)
        return
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_lutq(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
