"""Build libhqq.so in-tree for sm_100a (nvcc; no JIT cache, no torch extension).

    python weight_only_quantization_b200/build.py [--force]

(run as a file: importing the package loads the library this script builds)
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SOURCES = ["hqq_api.cu", "hqq_quantize.cu", "hqq_quantize_half.cu", "hqq_dequantize.cu", "hqq_meta.cu", "hqq_linear.cu", "hqq_decode.cu", "hqq_rtn.cu", "hqq_lowrank.cu"]
HEADERS = ["hqq_common.cuh", "hqq_params.cuh", "hqq_unpack.cuh", "hqq_quantize.cuh"]
LIB = os.path.join(PKG, "libhqq.so")

COMPILE_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    # binary32 arithmetic exactly as written: no contraction, IEEE div/sqrt, no FTZ
    "-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC,-ffp-contract=off,-fno-fast-math",
    "-Xptxas", "-v",
]
LINK_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static"]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "hqq.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source to an object in parallel (one nvcc per file), then
    link the shared library; the library is replaced only when all succeed."""
    if not (force or _stale()):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    objdir = tempfile.mkdtemp(prefix="hqq_build_")
    try:
        def compile_one(src: str):
            obj = os.path.join(objdir, os.path.splitext(src)[0] + ".o")
            cmd = ["nvcc", *COMPILE_FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
            return obj, subprocess.run(cmd, capture_output=True, text=True)
        workers = min(len(SOURCES), os.cpu_count() or 1)
        with ThreadPoolExecutor(max_workers=workers) as ex:
            results = list(ex.map(compile_one, SOURCES))
        log = "".join(r.stderr for _, r in results)
        for _, r in results:
            if r.returncode != 0:
                raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
        res = subprocess.run(["nvcc", *LINK_FLAGS, *[o for o, _ in results], "-o", tmp],
                             capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc link failed:\n" + res.stdout + res.stderr)
        if verbose:
            sys.stderr.write(log + res.stderr)
        os.replace(tmp, LIB)
    finally:
        shutil.rmtree(objdir, ignore_errors=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
