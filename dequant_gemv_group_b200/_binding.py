"""ctypes binding of liblutq (argument marshalling only).

Every function here forwards to the C ABI function of the same name declared
in ``include/lutq.h``; tensors are passed as raw device pointers, the stream is
torch's current CUDA stream.  There is no fallback: if ``liblutq.so`` is
missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# LUTQ_LIB_VARIANT=nvtx|bounds loads a tooling build of the same library
# (see build.py); the default is the product build
_VARIANT = os.environ.get("LUTQ_LIB_VARIANT") or None
LIB_PATH = os.path.join(_PKG, "liblutq.so" if _VARIANT is None else f"liblutq_{_VARIANT}.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python dequant_gemv_group_b200/build.py"
                      + (f" --variant {_VARIANT}`" if _VARIANT else "`"))

lib = ctypes.CDLL(LIB_PATH)

_i32, _i64, _vp = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p

LUTQ_OK = 0
STATUS_NAMES = {
    0: "LUTQ_OK", 1: "LUTQ_ERR_INVALID_ARG", 2: "LUTQ_ERR_SHAPE", 3: "LUTQ_ERR_BITS",
    4: "LUTQ_ERR_ALIGN", 5: "LUTQ_ERR_NONFINITE", 6: "LUTQ_ERR_CODE_RANGE",
    7: "LUTQ_ERR_TIMEOUT", 8: "LUTQ_ERR_CUDA", 9: "LUTQ_ERR_WORKSPACE", 10: "LUTQ_ERR_BOUNDS",
}
BUILD_NVTX, BUILD_BOUNDS = 1, 2
CODEBOOK_KINDS = {"nf4": 0, "logb": 1, "lloyd_max3": 2, "uniform4": 3}

_SIGS = {
    "lutq_status_string": (ctypes.c_char_p, [_i32]),
    "lutq_layout_version": (_i32, []),
    "lutq_build_flags": (_i32, []),
    "lutq_selftest_bounds": (_i32, [_vp, _vp]),
    "lutq_packed_bytes": (_i64, [_i64, _i64, _i32]),
    "lutq_codebook": (_i32, [_i32, _i32, _vp]),
    "lutq_quantize": (_i32, [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp]),
    "lutq_quantize_rowscale": (_i32, [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp]),
    "lutq_quantize_tensorscale": (_i32, [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp]),
    "lutq_quantize_group256": (_i32, [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp]),
    "lutq_codebook_asym_linear": (_i32, [ctypes.c_double, ctypes.c_double, _i32, _vp]),
    "lutq_pack": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp]),
    "lutq_workspace_bytes": (_i64, [_i64, _i64, _i64, _i32]),
    "lutq_workspace_zero_bytes": (_i64, [_i64, _i64, _i64, _i32]),
    "lutq_gemv": (_i32, [_vp, _i64, _vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _vp]),
    "lutq_gemm": (_i32, [_vp, _i64, _vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _vp]),
    "lutq_gemv_out_bf16": (_i32, [_vp, _i64, _vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp,
                                  _vp]),
    "lutq_gemm_out_bf16": (_i32, [_vp, _i64, _vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp,
                                  _vp]),
    "lutq_gemv_noalloc": (_i32, [_vp, _i64, _vp, _vp, _i32, _i64, _i64, _vp, _vp, _vp]),
    "lutq_gemv_plan": (_i32, [_i64, _i64, _i32, _vp]),
    "lutq_selftest_wait_timeout": (_i32, [_vp, _i64, _vp]),
    "lutq_fit_histogram": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "lutq_fit_codebook": (_i32, [_vp, _i32, _vp, _i32, _vp]),
    "lutq_rht_weights": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "lutq_rht_activations": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "lutq_gemv_rht": (_i32, [_vp, _i64, _vp, _vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp,
                             _vp]),
    "lutq_packed_bytes_group64": (_i64, [_i64, _i64, _i32]),
    "lutq_quantize_group64": (_i32, [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp]),
    "lutq_pack_group64": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp]),
    "lutq_gemv_group64": (_i32, [_vp, _i64, _vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp,
                                 _vp]),
    "lutq_gemm_group64": (_i32, [_vp, _i64, _vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp,
                                 _vp]),
    "lutq_max_types": (_i32, [_i32]),
    "lutq_packed_bytes_typed": (_i64, [_i64, _i64, _i32]),
    "lutq_quantize_typed": (_i32, [_vp, _i64, _i64, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "lutq_pack_typed": (_i32, [_vp, _vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp]),
    "lutq_gemv_typed": (_i32, [_vp, _i64, _vp, _vp, _i32, _i32, _i64, _i64, _vp, _vp, _i64, _vp,
                               _vp]),
    "lutq_gemm_typed": (_i32, [_vp, _i64, _vp, _vp, _i32, _i32, _i64, _i64, _vp, _vp, _i64, _vp,
                               _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class LutqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lutq_status_string(status)}")


def _check(status: int, where: str) -> None:
    if status != LUTQ_OK:
        raise LutqError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def lutq_status_string(status: int) -> str:
    return lib.lutq_status_string(int(status)).decode()


def lutq_layout_version() -> int:
    return lib.lutq_layout_version()


def lutq_build_flags() -> int:
    """BUILD_NVTX | BUILD_BOUNDS bits of the loaded library (0: product build)."""
    return int(lib.lutq_build_flags())


def lutq_selftest_bounds(status: torch.Tensor) -> None:
    """Run the kernels' index check on an index past its extent (see include/lutq.h)."""
    _need(status, torch.int32, "status")
    _check(lib.lutq_selftest_bounds(status.data_ptr(), _stream()), "lutq_selftest_bounds")


def lutq_packed_bytes(n: int, k: int, bits: int) -> int:
    return lib.lutq_packed_bytes(n, k, bits)


def lutq_workspace_bytes(m: int, n: int, k: int, bits: int) -> int:
    return lib.lutq_workspace_bytes(m, n, k, bits)


def lutq_workspace_zero_bytes(m: int, n: int, k: int, bits: int) -> int:
    return lib.lutq_workspace_zero_bytes(m, n, k, bits)


def lutq_gemv_plan(n: int, k: int, num_sms: int) -> dict:
    """How lutq_gemv divides an n x k problem among thread blocks (host only)."""
    out = (ctypes.c_int32 * 6)()
    _check(lib.lutq_gemv_plan(n, k, num_sms, out), "lutq_gemv_plan")
    return dict(zip(("C", "kind", "align", "Cm", "T", "nh"), list(out)))


def lutq_selftest_wait_timeout(status: torch.Tensor, limit_ns: int) -> None:
    """Run the kernels' bounded pipeline wait on a barrier nothing completes."""
    _need(status, torch.int32, "status")
    _check(lib.lutq_selftest_wait_timeout(status.data_ptr(), int(limit_ns), _stream()),
           "lutq_selftest_wait_timeout")


def lutq_codebook(kind: str, bits: int) -> torch.Tensor:
    """Host-built codebook as a CPU bf16 tensor of 2^bits ascending levels."""
    out = torch.zeros(1 << bits, dtype=torch.int16)
    _check(lib.lutq_codebook(CODEBOOK_KINDS[kind], bits, out.data_ptr()), "lutq_codebook")
    return out.view(torch.bfloat16)


def new_status(device=None) -> torch.Tensor:
    """A zeroed int32 device status word."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def new_workspace(m: int, n: int, k: int, bits: int, device=None) -> torch.Tensor:
    """A zero-filled workspace of lutq_workspace_bytes(m, n, k, bits) bytes."""
    nb = lutq_workspace_bytes(m, n, k, bits)
    if nb < 0:
        raise LutqError(2, "lutq_workspace_bytes")
    return torch.zeros(max(nb, 16), dtype=torch.uint8, device=device or "cuda")


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor of {dtype}")


def lutq_quantize(w: torch.Tensor, codebook: torch.Tensor, bits: int,
                  status: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    _need(w, torch.bfloat16, "W")
    _need(codebook, torch.bfloat16, "codebook")
    n, k = w.shape
    codes = torch.empty((n, k), dtype=torch.uint8, device=w.device)
    scales = torch.empty((n, max(k // 128, 1)), dtype=torch.bfloat16, device=w.device)
    _check(lib.lutq_quantize(w.data_ptr(), n, k, codebook.data_ptr(), bits, codes.data_ptr(),
                             scales.data_ptr(), _ptr(status), _stream()), "lutq_quantize")
    return codes, scales


def _quantize_scoped(fn, where, w, codebook, bits, status):
    _need(w, torch.bfloat16, "W")
    _need(codebook, torch.bfloat16, "codebook")
    n, k = w.shape
    codes = torch.empty((n, k), dtype=torch.uint8, device=w.device)
    scales = torch.empty((n, max(k // 128, 1)), dtype=torch.bfloat16, device=w.device)
    _check(fn(w.data_ptr(), n, k, codebook.data_ptr(), bits, codes.data_ptr(), scales.data_ptr(),
              _ptr(status), _stream()), where)
    return codes, scales


def lutq_quantize_rowscale(w: torch.Tensor, codebook: torch.Tensor, bits: int,
                           status: Optional[torch.Tensor] = None
                           ) -> Tuple[torch.Tensor, torch.Tensor]:
    """lutq_quantize with one scale per row (in every group's slot)."""
    return _quantize_scoped(lib.lutq_quantize_rowscale, "lutq_quantize_rowscale", w, codebook,
                            bits, status)


def lutq_quantize_group256(w: torch.Tensor, codebook: torch.Tensor, bits: int,
                           status: Optional[torch.Tensor] = None
                           ) -> Tuple[torch.Tensor, torch.Tensor]:
    """lutq_quantize with one scale per group of 256 (in both 128-group slots)."""
    return _quantize_scoped(lib.lutq_quantize_group256, "lutq_quantize_group256", w, codebook,
                            bits, status)


def lutq_quantize_tensorscale(w: torch.Tensor, codebook: torch.Tensor, bits: int,
                              status: Optional[torch.Tensor] = None
                              ) -> Tuple[torch.Tensor, torch.Tensor]:
    """lutq_quantize with one scale for the matrix (in every slot)."""
    return _quantize_scoped(lib.lutq_quantize_tensorscale, "lutq_quantize_tensorscale", w,
                            codebook, bits, status)


def lutq_codebook_asym_linear(w_min: float, w_max: float, bits: int) -> torch.Tensor:
    """The asymmetric linear codebook from w_min to w_max (bf16, host)."""
    out = torch.empty(1 << bits, dtype=torch.int16)
    _check(lib.lutq_codebook_asym_linear(float(w_min), float(w_max), bits, out.data_ptr()),
           "lutq_codebook_asym_linear")
    return out.view(torch.bfloat16)


def lutq_pack(codes: torch.Tensor, scales: torch.Tensor, bits: int,
              status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """codes uint8 [N, K] and scales bf16 [N, K/128] -> the packed matrix
    (layout V2, codes and scales); see lutq_pack in include/lutq.h."""
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.bfloat16, "scales")
    n, k = codes.shape
    if tuple(scales.shape) != (n, k // 128):
        raise LutqError(2, "lutq_pack: scales shape")
    nb = lutq_packed_bytes(n, k, bits)
    if nb < 0:
        raise LutqError(2, "lutq_packed_bytes")
    packed = torch.empty(nb, dtype=torch.uint8, device=codes.device)
    _check(lib.lutq_pack(codes.data_ptr(), scales.data_ptr(), n, k, bits, packed.data_ptr(),
                         _ptr(status), _stream()), "lutq_pack")
    return packed


def _product(fn, where, x, packed, codebook, bits, n, k, y, workspace, status,
             y_dtype=torch.float32):
    _need(x, torch.bfloat16, "x")
    m = x.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=y_dtype, device=x.device)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel())
    _check(fn(x.data_ptr(), m, packed.data_ptr(), codebook.data_ptr(), bits, n, k, y.data_ptr(),
              ws_ptr, ws_bytes, _ptr(status), _stream()), where)
    return y


def lutq_gemv(x, packed, codebook, bits, n, k, y=None, workspace=None, status=None):
    """y[M, N] (fp32) for M = 1..16; see lutq_gemv in include/lutq.h."""
    return _product(lib.lutq_gemv, "lutq_gemv", x, packed, codebook, bits, n, k, y, workspace,
                    status)


def lutq_gemv_out_bf16(x, packed, codebook, bits, n, k, y=None, workspace=None, status=None):
    """lutq_gemv writing y as bf16 (the fp32 sums rounded once)."""
    return _product(lib.lutq_gemv_out_bf16, "lutq_gemv_out_bf16", x, packed, codebook, bits, n,
                    k, y, workspace, status, torch.bfloat16)


def lutq_gemm_out_bf16(x, packed, codebook, bits, n, k, y=None, workspace=None, status=None):
    """lutq_gemm writing y as bf16 (the fp32 sums rounded once)."""
    return _product(lib.lutq_gemm_out_bf16, "lutq_gemm_out_bf16", x, packed, codebook, bits, n,
                    k, y, workspace, status, torch.bfloat16)


def lutq_gemv_noalloc(x, packed, codebook, bits, n, k, y=None, status=None):
    """lutq_gemv with the library's fixed scratch array instead of a workspace
    (for callers that cannot allocate device memory; see include/lutq.h)."""
    _need(x, torch.bfloat16, "x")
    m = x.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    _check(lib.lutq_gemv_noalloc(x.data_ptr(), m, packed.data_ptr(), codebook.data_ptr(), bits,
                                 n, k, y.data_ptr(), _ptr(status), _stream()),
           "lutq_gemv_noalloc")
    return y


def lutq_gemm(x, packed, codebook, bits, n, k, y=None, workspace=None, status=None):
    """y[M, N] (fp32) on the tensor cores; see lutq_gemm in include/lutq.h."""
    return _product(lib.lutq_gemm, "lutq_gemm", x, packed, codebook, bits, n, k, y, workspace,
                    status)


def _rht(fn, where, t: torch.Tensor, signs: torch.Tensor) -> torch.Tensor:
    _need(t, torch.bfloat16, where)
    _need(signs, torch.int8, "signs")
    if signs.numel() != 128:
        raise LutqError(1, where + ": 128 signs")
    rows, k = t.shape
    out = torch.empty_like(t)
    _check(fn(t.data_ptr(), rows, k, signs.data_ptr(), out.data_ptr(), _stream()), where)
    return out


def lutq_rht_weights(w: torch.Tensor, signs: torch.Tensor) -> torch.Tensor:
    """W bf16 [N, K] -> each 128-group rotated by H diag(s) (see include/lutq.h)."""
    return _rht(lib.lutq_rht_weights, "lutq_rht_weights", w, signs)


def lutq_rht_activations(x: torch.Tensor, signs: torch.Tensor) -> torch.Tensor:
    """x bf16 [M, K] -> each 128-group rotated by H diag(s) / 128."""
    return _rht(lib.lutq_rht_activations, "lutq_rht_activations", x, signs)


def lutq_gemv_rht(x, packed, codebook, signs, bits, n, k, y=None, workspace=None, status=None):
    """lutq_gemv on rotated weights, rotating x inside the kernel (M = 1..4)."""
    _need(x, torch.bfloat16, "x")
    _need(signs, torch.int8, "signs")
    m = x.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel())
    _check(lib.lutq_gemv_rht(x.data_ptr(), m, packed.data_ptr(), codebook.data_ptr(),
                             signs.data_ptr(), bits, n, k, y.data_ptr(), ws_ptr, ws_bytes,
                             _ptr(status), _stream()), "lutq_gemv_rht")
    return y


def lutq_packed_bytes_group64(n: int, k: int, bits: int) -> int:
    return int(lib.lutq_packed_bytes_group64(n, k, bits))


def lutq_quantize_group64(w: torch.Tensor, codebook: torch.Tensor, bits: int,
                          status: Optional[torch.Tensor] = None
                          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """W bf16 [N, K] -> (codes uint8 [N, K], scales bf16 [N, K/64]): one
    scale per group of 64 (see lutq_quantize_group64 in include/lutq.h)."""
    _need(w, torch.bfloat16, "W")
    _need(codebook, torch.bfloat16, "codebook")
    n, k = w.shape
    codes = torch.empty((n, k), dtype=torch.uint8, device=w.device)
    scales = torch.empty((n, max(k // 64, 1)), dtype=torch.bfloat16, device=w.device)
    _check(lib.lutq_quantize_group64(w.data_ptr(), n, k, codebook.data_ptr(), bits,
                                     codes.data_ptr(), scales.data_ptr(), _ptr(status),
                                     _stream()), "lutq_quantize_group64")
    return codes, scales


def lutq_pack_group64(codes: torch.Tensor, scales: torch.Tensor, bits: int,
                      status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """codes uint8 [N, K] and scales bf16 [N, K/64] -> the packed matrix with
    128-byte scale blocks."""
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.bfloat16, "scales")
    n, k = codes.shape
    if tuple(scales.shape) != (n, k // 64):
        raise LutqError(2, "lutq_pack_group64: scales shape")
    nb = lutq_packed_bytes_group64(n, k, bits)
    if nb < 0:
        raise LutqError(2, "lutq_packed_bytes_group64")
    packed = torch.empty(nb, dtype=torch.uint8, device=codes.device)
    _check(lib.lutq_pack_group64(codes.data_ptr(), scales.data_ptr(), n, k, bits,
                                 packed.data_ptr(), _ptr(status), _stream()),
           "lutq_pack_group64")
    return packed


def lutq_gemv_group64(x, packed, codebook, bits, n, k, y=None, workspace=None, status=None):
    """y[M, N] (fp32) with one scale per group of 64 (M = 1..16)."""
    return _product(lib.lutq_gemv_group64, "lutq_gemv_group64", x, packed, codebook, bits, n, k,
                    y, workspace, status)


def lutq_gemm_group64(x, packed, codebook, bits, n, k, y=None, workspace=None, status=None):
    """The group-64 product on the tensor cores (any M >= 1)."""
    return _product(lib.lutq_gemm_group64, "lutq_gemm_group64", x, packed, codebook, bits, n, k,
                    y, workspace, status)


def lutq_max_types(bits: int) -> int:
    return int(lib.lutq_max_types(bits))


def lutq_packed_bytes_typed(n: int, k: int, bits: int) -> int:
    return int(lib.lutq_packed_bytes_typed(n, k, bits))


def lutq_quantize_typed(w: torch.Tensor, codebooks: torch.Tensor, bits: int,
                        status: Optional[torch.Tensor] = None
                        ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """W bf16 [N, K] and codebooks bf16 [T, 2^bits] -> (codes uint8 [N, K],
    scales bf16 [N, K/128], group types uint8 [N, K/128]); see
    lutq_quantize_typed in include/lutq.h."""
    _need(w, torch.bfloat16, "W")
    _need(codebooks, torch.bfloat16, "codebooks")
    if codebooks.dim() != 2 or codebooks.shape[1] != (1 << bits):
        raise LutqError(3, "lutq_quantize_typed: codebooks must be [T, 2^bits]")
    n, k = w.shape
    g = max(k // 128, 1)
    codes = torch.empty((n, k), dtype=torch.uint8, device=w.device)
    scales = torch.empty((n, g), dtype=torch.bfloat16, device=w.device)
    types = torch.empty((n, g), dtype=torch.uint8, device=w.device)
    _check(lib.lutq_quantize_typed(w.data_ptr(), n, k, codebooks.data_ptr(), codebooks.shape[0],
                                   bits, codes.data_ptr(), scales.data_ptr(), types.data_ptr(),
                                   _ptr(status), _stream()), "lutq_quantize_typed")
    return codes, scales, types


def lutq_pack_typed(codes: torch.Tensor, scales: torch.Tensor, types: torch.Tensor, bits: int,
                    status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """codes, scales and group types -> the packed matrix with type blocks."""
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.bfloat16, "scales")
    _need(types, torch.uint8, "types")
    n, k = codes.shape
    if tuple(scales.shape) != (n, k // 128) or tuple(types.shape) != (n, k // 128):
        raise LutqError(2, "lutq_pack_typed: scales / types shape")
    nb = lutq_packed_bytes_typed(n, k, bits)
    if nb < 0:
        raise LutqError(2, "lutq_packed_bytes_typed")
    packed = torch.empty(nb, dtype=torch.uint8, device=codes.device)
    _check(lib.lutq_pack_typed(codes.data_ptr(), scales.data_ptr(), types.data_ptr(), n, k, bits,
                               packed.data_ptr(), _ptr(status), _stream()), "lutq_pack_typed")
    return packed


def _typed_product(fn, where, x, packed, codebooks, bits, n, k, y, workspace, status):
    _need(x, torch.bfloat16, "x")
    _need(codebooks, torch.bfloat16, "codebooks")
    m = x.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel())
    _check(fn(x.data_ptr(), m, packed.data_ptr(), codebooks.data_ptr(), codebooks.shape[0], bits,
              n, k, y.data_ptr(), ws_ptr, ws_bytes, _ptr(status), _stream()), where)
    return y


def lutq_gemv_typed(x, packed, codebooks, bits, n, k, y=None, workspace=None, status=None):
    """y[M, N] (fp32) with per-group types, codebooks bf16 [T, 2^bits]
    (M = 1..16; see lutq_gemv_typed in include/lutq.h)."""
    return _typed_product(lib.lutq_gemv_typed, "lutq_gemv_typed", x, packed, codebooks, bits,
                          n, k, y, workspace, status)


def lutq_gemm_typed(x, packed, codebooks, bits, n, k, y=None, workspace=None, status=None):
    """The typed product on the tensor cores (any M >= 1)."""
    return _typed_product(lib.lutq_gemm_typed, "lutq_gemm_typed", x, packed, codebooks, bits,
                          n, k, y, workspace, status)


HIST_BINS = 16384


def lutq_fit_histogram(w: torch.Tensor, hist: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Add W's normalised-weight counts to hist (int64 [16384] on W's device,
    zeros if None) and return it."""
    _need(w, torch.bfloat16, "W")
    n, k = w.shape
    if hist is None:
        hist = torch.zeros(HIST_BINS, dtype=torch.int64, device=w.device)
    _need(hist, torch.int64, "hist")
    _check(lib.lutq_fit_histogram(w.data_ptr(), n, k, hist.data_ptr(), _ptr(status), _stream()),
           "lutq_fit_histogram")
    return hist


def lutq_fit_codebook(hist, bits: int, init: torch.Tensor, max_iter: int = 100) -> torch.Tensor:
    """Lloyd-Max from init (bf16, CPU) on a histogram (CPU, from
    lutq_fit_histogram); returns the fitted codebook (bf16, CPU)."""
    h = torch.as_tensor(hist).to(device="cpu", dtype=torch.int64).contiguous()
    if h.numel() != HIST_BINS:
        raise LutqError(1, "lutq_fit_codebook: histogram size")
    init_c = init.to(device="cpu", dtype=torch.bfloat16).contiguous()
    out = torch.empty(1 << bits, dtype=torch.bfloat16)
    _check(lib.lutq_fit_codebook(h.data_ptr(), bits, init_c.data_ptr(), max_iter, out.data_ptr()),
           "lutq_fit_codebook")
    return out
