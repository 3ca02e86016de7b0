"""Seeded synthetic inputs for the LUT-quantized GEMV/GEMM workloads.

This module draws random numbers and nothing else: it holds none of the
quantization, packing or product arithmetic.  Both the CPU oracle side (tests,
CPU baseline) and the CUDA library side (tests, bench) take their inputs from
here, so that the two are compared on identical tensors.

Recipe (one rule for every workload):
  * all draws come from one ``torch.Generator`` seeded per tensor (weights use
    the workload's weight seed, activations the activation seed);
  * draws are made in fp32, scaled, outliers are applied in fp32, and the
    result is cast to bf16 exactly once (round to nearest even);
  * "0.1% entries x10 outliers" means exactly round(1e-3 * N * K) distinct
    positions, taken as the first entries of a seeded permutation of all
    N*K positions, multiplied by 10 before the cast;
  * Student-t(nu) is Z / sqrt(chi2_nu / nu) with chi2_nu the sum of nu
    squared standard normals, all from the same generator;
  * weights are drawn in row chunks of ``_CHUNK_ROWS`` rows so that peak host
    memory stays bounded for the 70B-shaped layers; the chunking is part of
    the definition and therefore fixed.

The shapes and distributions follow the five workloads of the LUT-quantized
LLM layer study (Llama-3 8B/70B-shaped linear layers, batch 1..128).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import torch

_CHUNK_ROWS = 2048

# Codebook kinds (mirrors the integer ids of the C ABI; only names live here).
NF4 = "nf4"
LOGB = "logb"
LM3 = "lloyd_max3"
UNIFORM4 = "uniform4"


def _normal_chunked(n: int, k: int, gen: torch.Generator) -> torch.Tensor:
    out = torch.empty((n, k), dtype=torch.float32)
    for r0 in range(0, n, _CHUNK_ROWS):
        r1 = min(n, r0 + _CHUNK_ROWS)
        out[r0:r1] = torch.randn((r1 - r0, k), generator=gen, dtype=torch.float32)
    return out


def _apply_outliers(w: torch.Tensor, frac: float, gen: torch.Generator) -> None:
    if frac <= 0.0:
        return
    total = w.numel()
    count = int(round(frac * total))
    if count == 0:
        return
    pos = torch.randperm(total, generator=gen)[:count]
    flat = w.view(-1)
    flat[pos] = flat[pos] * 10.0


def normal_weights(n: int, k: int, std: float, seed: int,
                   outlier_frac: float = 0.0) -> torch.Tensor:
    """W[n,k] ~ N(0, std^2), optional outliers, as bf16 on the CPU."""
    gen = torch.Generator().manual_seed(seed)
    w = _normal_chunked(n, k, gen)
    w.mul_(std)
    _apply_outliers(w, outlier_frac, gen)
    return w.to(torch.bfloat16)


def student_t_weights(n: int, k: int, nu: int, scale: float, seed: int,
                      outlier_frac: float = 0.0) -> torch.Tensor:
    """W[n,k] ~ scale * Student-t(nu), as bf16 on the CPU."""
    gen = torch.Generator().manual_seed(seed)
    out = torch.empty((n, k), dtype=torch.float32)
    for r0 in range(0, n, _CHUNK_ROWS):
        r1 = min(n, r0 + _CHUNK_ROWS)
        z = torch.randn((r1 - r0, k), generator=gen, dtype=torch.float32)
        chi2 = torch.zeros_like(z)
        for _ in range(nu):
            e = torch.randn((r1 - r0, k), generator=gen, dtype=torch.float32)
            chi2.addcmul_(e, e)
        out[r0:r1] = z / torch.sqrt(chi2 / float(nu))
    out.mul_(scale)
    _apply_outliers(out, outlier_frac, gen)
    return out.to(torch.bfloat16)


def activations(m: int, k: int, seed: int) -> torch.Tensor:
    """x[m,k] ~ N(0,1), as bf16 on the CPU."""
    gen = torch.Generator().manual_seed(seed)
    return torch.randn((m, k), generator=gen, dtype=torch.float32).to(torch.bfloat16)


def rht_signs(seed: int) -> torch.Tensor:
    """128 random signs (+1 / -1, int8) for the randomized Hadamard rotation."""
    gen = torch.Generator().manual_seed(seed)
    return (torch.randint(0, 2, (128,), generator=gen) * 2 - 1).to(torch.int8)


@dataclasses.dataclass(frozen=True)
class Layer:
    """One weight matrix of a workload: W[n, k] and how it is drawn."""
    name: str
    n: int
    k: int
    dist: str            # "normal" or "student_t"
    std: float           # std (normal) or scale (student_t)
    outlier_frac: float = 0.0
    nu: int = 5

    def weights(self, seed: int = 0) -> torch.Tensor:
        if self.dist == "normal":
            return normal_weights(self.n, self.k, self.std, seed, self.outlier_frac)
        if self.dist == "student_t":
            return student_t_weights(self.n, self.k, self.nu, self.std, seed,
                                     self.outlier_frac)
        raise ValueError(self.dist)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    layers: Tuple[Layer, ...]
    codebooks: Tuple[Tuple[str, int], ...]   # (codebook kind, bits)
    batches: Tuple[int, ...]
    weight_seed: int = 0
    act_seed: int = 1


WORKLOADS: Dict[str, Workload] = {
    # Tiny W4 NF4 GEMV, 1024x1024, N(0,0.02) with 0.1% x10 outliers, batch 1.
    "tiny_w4_nf4": Workload(
        "tiny_w4_nf4",
        (Layer("w", 1024, 1024, "normal", 0.02, 1e-3),),
        ((NF4, 4),), (1,)),
    # W3 plain LUT GEMV: Lloyd-Max 8-level codebook, 4096x4096 N(0,0.02), batch 1.
    "w3_lm3_4096": Workload(
        "w3_lm3_4096",
        (Layer("w", 4096, 4096, "normal", 0.02),),
        ((LM3, 3),), (1,)),
    # W4 log-base codebook (b=1.6), 14336x4096 Student-t(5)*0.02, batch 1/4/8.
    "w4_logb_14336x4096": Workload(
        "w4_logb_14336x4096",
        (Layer("w", 14336, 4096, "student_t", 0.02),),
        ((LOGB, 4),), (1, 4, 8)),
    # Llama-3-8B-shaped layer set, W4 NF4, N(0,0.02) with 0.1% outliers.
    "llama3_8b_w4_nf4": Workload(
        "llama3_8b_w4_nf4",
        (Layer("q_o", 4096, 4096, "normal", 0.02, 1e-3),
         Layer("k_v", 1024, 4096, "normal", 0.02, 1e-3),
         Layer("gate_up", 14336, 4096, "normal", 0.02, 1e-3),
         Layer("down", 4096, 14336, "normal", 0.02, 1e-3)),
        ((NF4, 4),), (1, 2, 4, 8, 16)),
    # 70B-shaped MLP, W4 NF4 and W3 Lloyd-Max, N(0,0.015), batch 1..128.
    "llama3_70b_mlp": Workload(
        "llama3_70b_mlp",
        (Layer("gate_up", 28672, 8192, "normal", 0.015),
         Layer("down", 8192, 28672, "normal", 0.015)),
        ((NF4, 4), (LM3, 3)), (1, 2, 4, 8, 16, 32, 64, 128)),
}


def layer(workload: str, name: str) -> Layer:
    for lay in WORKLOADS[workload].layers:
        if lay.name == name:
            return lay
    raise KeyError(f"{workload}/{name}")


def all_cases() -> List[Tuple[str, Layer, str, int, int]]:
    """Every (workload, layer, codebook kind, bits, batch) combination."""
    out = []
    for wl in WORKLOADS.values():
        for lay in wl.layers:
            for kind, bits in wl.codebooks:
                for m in wl.batches:
                    out.append((wl.name, lay, kind, bits, m))
    return out
