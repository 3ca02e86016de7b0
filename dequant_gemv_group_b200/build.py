"""Build liblutq.so (the CUDA kernels and the C ABI) in-tree for sm_100a.

Run as ``python dequant_gemv_group_b200/build.py`` (the package itself needs the
library to import) or call :func:`build`.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblutq.so")
BUILD_DIR = os.path.join(ROOT, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
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


def _run(cmd, log):
    r = subprocess.run(cmd, capture_output=True, text=True)
    log.write(" ".join(cmd) + "\n" + r.stdout + r.stderr + "\n")
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("build failed: " + " ".join(cmd))


def _stale(objs) -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "lutq.h"),
                                                               os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    objs = []
    if not force and not _stale(objs):
        return LIB
    log_path = os.path.join(BUILD_DIR, "build.log")
    with open(log_path, "w") as log:
        for src in SOURCES:
            obj = os.path.join(BUILD_DIR, src + ".o")
            _run([NVCC, *ARCH, *COMMON, *PER_FILE.get(src, []), "-c",
                  os.path.join(CSRC, src), "-o", obj], log)
            objs.append(obj)
        for src in HOST_SOURCES:
            obj = os.path.join(BUILD_DIR, src + ".o")
            _run(["g++", "-O2", "-std=c++17", "-fPIC", "-I", INCLUDE, "-c",
                  os.path.join(CSRC, src), "-o", obj], log)
            objs.append(obj)
        tmp = LIB + ".tmp"
        _run([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-ldl", "-lrt",
              "-lpthread"], log)
        os.replace(tmp, LIB)
    if verbose:
        print(open(log_path).read())
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
