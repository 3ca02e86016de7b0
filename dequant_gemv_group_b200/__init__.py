"""Group-wise lookup-table weight quantization and fused dequant GEMV/GEMM for
NVIDIA B200 (sm_100a).

The work is done by ``liblutq.so`` (CUDA kernels behind a C ABI, declared in
``include/lutq.h``); this package only marshals torch tensors into it.
"""
from ._binding import (  # noqa: F401
    CODEBOOK_KINDS,
    HIST_BINS,
    LIB_PATH,
    LutqError,
    lib,
    lutq_codebook,
    lutq_codebook_asym_linear,
    lutq_fit_codebook,
    lutq_fit_histogram,
    lutq_gemm,
    lutq_gemm_out_bf16,
    lutq_gemm_typed,
    lutq_gemv,
    lutq_gemv_noalloc,
    lutq_gemv_out_bf16,
    lutq_gemv_plan,
    lutq_gemv_rht,
    lutq_gemv_typed,
    lutq_layout_version,
    lutq_max_types,
    lutq_pack,
    lutq_pack_typed,
    lutq_packed_bytes,
    lutq_packed_bytes_typed,
    lutq_quantize,
    lutq_quantize_group256,
    lutq_quantize_rowscale,
    lutq_quantize_tensorscale,
    lutq_quantize_typed,
    lutq_rht_activations,
    lutq_rht_weights,
    lutq_selftest_wait_timeout,
    lutq_status_string,
    lutq_workspace_bytes,
    new_status,
    new_workspace,
)
