"""Build libhqq.so in-tree for sm_100a (nvcc; no JIT cache, no torch extension).

    python weight_only_quantization_b200/build.py [--force]

(run as a file: importing the package loads the library this script builds)
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SOURCES = ["hqq_api.cu", "hqq_quantize.cu", "hqq_dequantize.cu", "hqq_meta.cu", "hqq_linear.cu", "hqq_decode.cu", "hqq_rtn.cu", "hqq_lowrank.cu"]
HEADERS = ["hqq_common.cuh", "hqq_params.cuh", "hqq_unpack.cuh"]
LIB = os.path.join(PKG, "libhqq.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    # binary32 arithmetic exactly as written: no contraction, IEEE div/sqrt, no FTZ
    "-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC,-ffp-contract=off,-fno-fast-math",
    "-Xptxas", "-v",
    "-shared", "-cudart", "static",
]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "hqq.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not (force or _stale()):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["nvcc", *NVCC_FLAGS, *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
