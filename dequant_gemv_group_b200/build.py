"""Build liblutq.so (the CUDA kernels and the C ABI) in-tree for sm_100a.

Run as ``python dequant_gemv_group_b200/build.py [--variant nvtx|bounds]
[--force] [-v]`` (the package itself needs the library to import) or call
:func:`build`.  Variants are separate libraries beside the default one:

  liblutq.so         the product;
  liblutq_nvtx.so    -DLUTQ_NVTX: every C-ABI call opens an NVTX range;
  liblutq_bounds.so  -DLUTQ_BOUNDS: the kernels check their indices against
                     the buffers' extents and report LUTQ_ERR_BOUNDS.

The binding loads the default library unless LUTQ_LIB_VARIANT names a variant.
Sources compile in parallel; ptxas' register, spill and shared-memory report
(-Xptxas -v) goes to _build/<variant>/build.log.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblutq.so")
BUILD_DIR = os.path.join(ROOT, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
CUDA_INCLUDE = os.path.join(os.path.dirname(os.path.dirname(NVCC)), "include")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
          "-Xptxas", "-v"]
# The quantizer must use the IEEE divide and no contraction or flush-to-zero.
PER_FILE = {
    "lutq_quantize.cu": ["-fmad=false", "-ftz=false", "-prec-div=true", "-prec-sqrt=true"],
}
SOURCES = ["lutq_api.cu", "lutq_quantize.cu", "lutq_pack.cu", "lutq_gemv.cu", "lutq_gemm.cu",
           "lutq_noalloc.cu", "lutq_selftest.cu", "lutq_rht.cu", "lutq_fit.cu"]
HOST_SOURCES = ["lutq_codebook.cpp"]
VARIANTS = {None: [], "nvtx": ["-DLUTQ_NVTX"], "bounds": ["-DLUTQ_BOUNDS"]}


def lib_path(variant: str | None = None) -> str:
    return LIB if variant is None else os.path.join(PKG, f"liblutq_{variant}.so")


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    return cmd, r.returncode, r.stdout + r.stderr


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "lutq.h"),
                                                               os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, variant: str | None = None) -> str:
    if variant not in VARIANTS:
        raise ValueError(f"unknown variant {variant!r}")
    lib = lib_path(variant)
    if not force and not _stale(lib):
        return lib
    flags = VARIANTS[variant]
    bdir = os.path.join(BUILD_DIR, variant or "default")
    os.makedirs(bdir, exist_ok=True)
    jobs, objs = [], []
    for src in SOURCES:
        obj = os.path.join(bdir, src + ".o")
        jobs.append([NVCC, *ARCH, *COMMON, *flags, *PER_FILE.get(src, []), "-c",
                     os.path.join(CSRC, src), "-o", obj])
        objs.append(obj)
    for src in HOST_SOURCES:
        obj = os.path.join(bdir, src + ".o")
        jobs.append(["g++", "-O2", "-std=c++17", "-fPIC", *flags, "-I", INCLUDE, "-I", CUDA_INCLUDE,
                     "-c", os.path.join(CSRC, src), "-o", obj])
        objs.append(obj)
    log_path = os.path.join(bdir, "build.log")
    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as pool:
        results = list(pool.map(_run, jobs))
    tmp = lib + ".tmp"
    if all(rc == 0 for _, rc, _ in results):
        results.append(_run([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-ldl",
                             "-lrt", "-lpthread"]))
    with open(log_path, "w") as log:
        for cmd, rc, out in results:
            log.write(" ".join(cmd) + "\n" + out + "\n")
    failed = [(cmd, out) for cmd, rc, out in results if rc != 0]
    if failed:
        cmd, out = failed[0]
        sys.stderr.write(out)
        raise RuntimeError("build failed: " + " ".join(cmd))
    os.replace(tmp, lib)
    if verbose:
        print(open(log_path).read())
    return lib


if __name__ == "__main__":
    v = None
    if "--variant" in sys.argv:
        v = sys.argv[sys.argv.index("--variant") + 1]
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, variant=v))
