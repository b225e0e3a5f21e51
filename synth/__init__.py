"""Seeded synthetic LLM-like weight matrices (input generator only).

Shared by the tests, the benchmark and the smoke check; it holds none of the
quantization method's arithmetic.  Both generators draw the same Philox4x32-10
uniforms (Salmon et al., SC'11; counter = (index lo, index hi, draw, 0), key =
(seed, stream)) and map them to Student-t(4) scaled to ``std``, with a fraction
``outlier_frac`` of entries multiplied by ``outlier_mult``, rounded to fp16.
The host (numpy, float64 transforms) and device (CUDA, float32 transforms)
versions agree on the draws; their fp16 values may differ in the last bit.

Workload recipe (shapes of the Llama-2 family quoted for the method's timings):
  * single matrices 1024x1024 (seed 0) and 4096x4096 (seed 1);
  * a 7B-shaped set: 32 layers x {q,k,v,o 4096x4096; gate,up 11008x4096;
    down 4096x11008} (seed 2);
  * two 70B-shaped matrices 8192x8192 and 28672x8192 (seed 3);
  * a 70B-shaped set: 80 layers x {q,o 8192x8192; k,v 1024x8192;
    gate,up 28672x8192; down 8192x28672} (seed 5).
  Matrix m of layer l uses stream id 7*l + m (m in q,k,v,o,gate,up,down order).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

STD = 0.02
OUTLIER_FRAC = 1e-3
OUTLIER_MULT = 20.0

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.cu")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None

MATRIX_ORDER = ("q", "k", "v", "o", "gate", "up", "down")


def llama2_7b_shapes():
    """(out, in) of each linear matrix of one Llama-2-7B-shaped layer."""
    h, f = 4096, 11008
    return {"q": (h, h), "k": (h, h), "v": (h, h), "o": (h, h),
            "gate": (f, h), "up": (f, h), "down": (h, f)}


def llama2_70b_shapes():
    """(out, in) of each linear matrix of one Llama-2-70B-shaped layer (GQA k/v)."""
    h, f, kv = 8192, 28672, 1024
    return {"q": (h, h), "k": (kv, h), "v": (kv, h), "o": (h, h),
            "gate": (f, h), "up": (f, h), "down": (h, f)}


def stream_id(layer: int, name: str) -> int:
    return 7 * layer + MATRIX_ORDER.index(name)


# --------------------------------------------------------------------------- host
_M0, _M1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
_W0, _W1 = np.uint32(0x9E3779B9), np.uint32(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Vectorised Philox4x32-10 over uint32 counter arrays; returns 4 arrays."""
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint32) for c in (c0, c1, c2, c3))
    k0 = np.uint32(k0)
    k1 = np.uint32(k1)
    with np.errstate(over="ignore"):
        for _ in range(10):
            p0 = _M0 * c0.astype(np.uint64)
            p1 = _M1 * c2.astype(np.uint64)
            hi0, lo0 = (p0 >> np.uint64(32)).astype(np.uint32), (p0 & _MASK).astype(np.uint32)
            hi1, lo1 = (p1 >> np.uint64(32)).astype(np.uint32), (p1 & _MASK).astype(np.uint32)
            c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
            k0 = np.uint32(k0 + _W0)
            k1 = np.uint32(k1 + _W1)
    return c0, c1, c2, c3


def _unit_open(x):
    return ((x >> np.uint32(8)).astype(np.float64) + 0.5) * (1.0 / 16777216.0)


def student_t_host(shape, seed: int, stream: int = 0, std: float = STD,
                   outlier_frac: float = OUTLIER_FRAC, outlier_mult: float = OUTLIER_MULT,
                   start: int = 0) -> np.ndarray:
    """fp16 array of the given shape (flat elements start..start+n)."""
    n = int(np.prod(shape))
    idx = np.arange(start, start + n, dtype=np.uint64)
    lo = (idx & _MASK).astype(np.uint32)
    hi = (idx >> np.uint64(32)).astype(np.uint32)
    zero = np.zeros(n, np.uint32)
    a = philox4x32_10(lo, hi, zero, zero, seed, stream)
    b = philox4x32_10(lo, hi, zero + 1, zero, seed, stream)
    zn = np.sqrt(-2.0 * np.log(_unit_open(a[0]))) * np.cos(2.0 * np.pi * _unit_open(a[1]))
    chi2 = -2.0 * (np.log(_unit_open(a[2])) + np.log(_unit_open(a[3])))
    v = zn / np.sqrt(chi2 * 0.25) * (std / np.sqrt(2.0))
    th = np.uint32(min(max(outlier_frac * 4294967296.0, 0), 4294967295.0))
    v = np.where(b[0] < th, v * outlier_mult, v)
    return v.astype(np.float16).reshape(shape)


# ------------------------------------------------------------------------- device
def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                        "-std=c++17", "-Xcompiler", "-fPIC", "-shared", _SRC, "-o", tmp],
                       check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.synth_student_t_fp16.argtypes = [ctypes.c_void_p, ctypes.c_int64,
                                                 ctypes.c_uint32, ctypes.c_uint32,
                                                 ctypes.c_float, ctypes.c_double,
                                                 ctypes.c_float, ctypes.c_void_p]
            lib.synth_student_t_fp16.restype = ctypes.c_int
            _lib = lib
    return _lib


def fill_student_t_(t, seed: int, stream: int = 0, std: float = STD,
                    outlier_frac: float = OUTLIER_FRAC,
                    outlier_mult: float = OUTLIER_MULT):
    """Fill a contiguous fp16 CUDA tensor in place on the current stream."""
    import torch
    assert t.is_cuda and t.dtype == torch.float16 and t.is_contiguous()
    st = _load().synth_student_t_fp16(ctypes.c_void_p(t.data_ptr()), t.numel(), seed,
                                      stream, std, outlier_frac, outlier_mult,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if st:
        raise RuntimeError(f"synth_student_t_fp16 failed with status {st}")
    return t


def student_t_device(shape, seed: int, stream: int = 0, device="cuda", **kw):
    import torch
    t = torch.empty(shape, dtype=torch.float16, device=device)
    return fill_student_t_(t, seed, stream, **kw)
