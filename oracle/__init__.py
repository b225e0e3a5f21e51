"""CPU oracle for group-wise HQQ quantization -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``hqq_oracle.c`` (plain scalar
fp32, see the header comment of that file for the method, its source sections
and the readings taken) through ctypes.  Three functions are plain numpy in
fp64 instead: ``linear`` (the product with the dequantized weights),
``quant_error`` (W - W_hat) and ``lowrank`` (the truncated SVD of the
quantization error).  It shares no code with the CUDA path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hqq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhqq_oracle.so")
_CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-pthread"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle library in-tree (gcc, strict IEEE fp32)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I64, I, F = ctypes.c_int64, ctypes.c_int, ctypes.c_float
            lib.hqq_oracle_quantize.argtypes = [P, I64, I, I, F, F, F, I, I, P, P, P, P, P, P, P]
            lib.hqq_oracle_quantize.restype = I
            lib.hqq_oracle_trace_group.argtypes = [P, I, I, F, F, F, I, P, P, P, P, P, P, P, P, P]
            lib.hqq_oracle_trace_group.restype = I
            lib.hqq_oracle_quantize_half.argtypes = [P, I64, I, I, F, F, F, I, I, P, P, P, P, P,
                                                     P, P, P]
            lib.hqq_oracle_quantize_half.restype = I
            lib.hqq_oracle_trace_group_half.argtypes = [P, I, I, F, F, F, I, P, P, P, P, P, P,
                                                        P, P, P]
            lib.hqq_oracle_trace_group_half.restype = I
            lib.hqq_oracle_shrink.argtypes = [P, I64, F, F, P]
            lib.hqq_oracle_shrink.restype = None
            lib.hqq_oracle_z_update.argtypes = [P, P, P, I, F]
            lib.hqq_oracle_z_update.restype = F
            lib.hqq_oracle_powp.argtypes = [P, I64, F, P]
            lib.hqq_oracle_powp.restype = None
            lib.hqq_oracle_powp_table.argtypes = [F, P, P, P, P]
            lib.hqq_oracle_powp_table.restype = None
            lib.hqq_oracle_psum.argtypes = [P, I]
            lib.hqq_oracle_psum.restype = F
            lib.hqq_oracle_packed_bytes.argtypes = [I64, I]
            lib.hqq_oracle_packed_bytes.restype = I64
            lib.hqq_oracle_pack.argtypes = [P, I64, I, P]
            lib.hqq_oracle_pack.restype = I
            lib.hqq_oracle_unpack.argtypes = [P, I64, I, P]
            lib.hqq_oracle_unpack.restype = I
            lib.hqq_oracle_dequantize.argtypes = [P, P, P, I64, I, P]
            lib.hqq_oracle_dequantize.restype = I
            lib.hqq_oracle_f32_to_f16.argtypes = [P, I64, P]
            lib.hqq_oracle_f32_to_f16.restype = None
            lib.hqq_oracle_meta_quantize.argtypes = [P, I64, I64, P, P, P]
            lib.hqq_oracle_meta_quantize.restype = I
            lib.hqq_oracle_meta_dequantize.argtypes = [P, P, P, I64, I64, P]
            lib.hqq_oracle_meta_dequantize.restype = I
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


DEFAULTS = dict(p=0.7, beta=1.0, kappa=1.01, iters=20)


def quantize(W: np.ndarray, nbits: int, group: int, p: float = 0.7, beta: float = 1.0,
             kappa: float = 1.01, iters: int = 20, threads: int | None = None,
             precision: str = "fp32") -> dict:
    """HQQ-quantize an fp16 array (any shape, flat size a multiple of ``group``;
    groups are contiguous runs of ``group`` elements of the flat row-major order).

    ``precision`` "fp32": the single-precision solver; "fp16": the half-precision
    solver (groups outside its fp16 bounds solved in single precision; ``half``
    in the result marks the groups solved in fp16).

    Returns codes (uint8 per weight, flat), packed bytes, fp16 scale/zero per
    group, the fp32 zero and scale, the accepted minimum of the error (the
    binary32 sum; the fp16 mean for groups solved in half precision; +inf when
    iters = 0) and the accepted-iteration count per group.
    """
    if precision not in ("fp32", "fp16"):
        raise ValueError("precision must be 'fp32' or 'fp16'")
    lib = _load()
    W = np.ascontiguousarray(W, dtype=np.float16).reshape(-1)
    n = W.size
    if n % group:
        raise ValueError("size must be a multiple of the group size")
    ng = n // group
    codes = np.empty(n, np.uint8)
    scale = np.empty(ng, np.uint16)
    zero = np.empty(ng, np.uint16)
    zf = np.empty(ng, np.float32)
    sf = np.empty(ng, np.float32)
    it = np.empty(ng, np.uint8)
    err = np.empty(ng, np.float32)
    if threads is None:
        threads = os.cpu_count() or 1
    half = np.zeros(ng, np.uint8)
    if precision == "fp32":
        st = lib.hqq_oracle_quantize(_ptr(W.view(np.uint16)), ng, group, nbits, p, beta, kappa,
                                     iters, threads, _ptr(codes), _ptr(scale), _ptr(zero),
                                     _ptr(zf), _ptr(sf), _ptr(err), _ptr(it))
    else:
        st = lib.hqq_oracle_quantize_half(_ptr(W.view(np.uint16)), ng, group, nbits, p, beta,
                                          kappa, iters, threads, _ptr(codes), _ptr(scale),
                                          _ptr(zero), _ptr(zf), _ptr(sf), _ptr(err), _ptr(it),
                                          _ptr(half))
    if st:
        raise ValueError(f"oracle rejected the arguments (status {st})")
    return dict(codes=codes, packed=pack(codes, nbits), scale=scale.view(np.float16),
                zero=zero.view(np.float16), zero_f32=zf, scale_f32=sf, err=err, iters=it,
                half=half.astype(bool))


def trace_group(w, nbits: int, p: float = 0.7, beta: float = 1.0, kappa: float = 1.01,
                iters: int = 20, precision: str = "fp32") -> dict:
    """Solve one group (fp32 values; for "fp16" they must be fp16 values) and
    return its whole per-iteration record; ``half`` tells whether the
    half-precision solver took the group."""
    if precision not in ("fp32", "fp16"):
        raise ValueError("precision must be 'fp32' or 'fp16'")
    lib = _load()
    w = np.ascontiguousarray(w, dtype=np.float32)
    G = w.size
    T = max(iters, 1)
    codes = np.empty(G, np.uint8)
    out6 = np.empty(6, np.float32)
    counts = np.zeros(3, np.int32)
    z = np.full(T, np.nan, np.float32)
    e = np.full(T, np.nan, np.float32)
    bh = np.full(T, np.nan, np.float32)
    q = np.full((T, G), np.nan, np.float32)
    d = np.full((T, G), np.nan, np.float32)
    we = np.full((T, G), np.nan, np.float32)
    fn = lib.hqq_oracle_trace_group if precision == "fp32" else lib.hqq_oracle_trace_group_half
    st = fn(_ptr(w), G, nbits, p, beta, kappa, iters, _ptr(codes), _ptr(out6), _ptr(counts),
            _ptr(z), _ptr(e), _ptr(bh), _ptr(q), _ptr(d), _ptr(we))
    if st:
        raise ValueError(f"oracle rejected the arguments (status {st})")
    ne = int(counts[1])
    return dict(codes=codes, s=out6[0], inv=out6[1], z0=out6[2], z_best=out6[3],
                e_best=out6[4], accepted=int(counts[0]), evaluations=ne,
                half=bool(counts[2]),
                z=z[:ne], e=e[:ne], beta=bh[:ne], q=q[:ne], d=d[:ne], we=we[:ne])


def shrink(x, p: float, beta: float) -> np.ndarray:
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty_like(x)
    lib.hqq_oracle_shrink(_ptr(x), x.size, p, beta, _ptr(out))
    return out


def z_update(w, q, we, inv: float) -> np.float32:
    lib = _load()
    w = np.ascontiguousarray(w, dtype=np.float32)
    q = np.ascontiguousarray(q, dtype=np.float32)
    we = np.ascontiguousarray(we, dtype=np.float32)
    return np.float32(lib.hqq_oracle_z_update(_ptr(w), _ptr(q), _ptr(we), w.size, inv))


def powp(x, p: float) -> np.ndarray:
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty_like(x)
    lib.hqq_oracle_powp(_ptr(x), x.size, p, _ptr(out))
    return out


def powp_table(p: float) -> dict:
    lib = _load()
    a = np.empty(256, np.float32)
    b = np.empty(32, np.float32)
    c = np.empty(32, np.float32)
    k = np.empty(3, np.float32)
    lib.hqq_oracle_powp_table(p, _ptr(a), _ptr(b), _ptr(c), _ptr(k))
    return dict(two_pk=a, cj_p=b, inv_cj=c, coef=k)


def psum(x) -> np.float32:
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    return np.float32(lib.hqq_oracle_psum(_ptr(x), x.size))


def packed_bytes(n: int, nbits: int) -> int:
    return int(_load().hqq_oracle_packed_bytes(n, nbits))


def pack(codes, nbits: int) -> np.ndarray:
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8).reshape(-1)
    out = np.empty(packed_bytes(codes.size, nbits), np.uint8)
    st = lib.hqq_oracle_pack(_ptr(codes), codes.size, nbits, _ptr(out))
    if st:
        raise ValueError(f"pack failed (status {st})")
    return out


def unpack(packed, n: int, nbits: int) -> np.ndarray:
    lib = _load()
    packed = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    if packed.size < packed_bytes(n, nbits):
        raise ValueError("packed buffer too small")
    out = np.empty(n, np.uint8)
    st = lib.hqq_oracle_unpack(_ptr(packed), n, nbits, _ptr(out))
    if st:
        raise ValueError(f"unpack failed (status {st})")
    return out


def dequantize(codes, scale, zero, group: int) -> np.ndarray:
    """W_hat = fp16((c - z) * s) per element, s and z the stored fp16 values."""
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8).reshape(-1)
    scale = np.ascontiguousarray(scale, dtype=np.float16).reshape(-1)
    zero = np.ascontiguousarray(zero, dtype=np.float16).reshape(-1)
    out = np.empty(codes.size, np.uint16)
    st = lib.hqq_oracle_dequantize(_ptr(codes), _ptr(scale.view(np.uint16)),
                                   _ptr(zero.view(np.uint16)), codes.size, group, _ptr(out))
    if st:
        raise ValueError(f"dequantize failed (status {st})")
    return out.view(np.float16)


def meta_groups(n: int, group: int) -> int:
    """Number of groups of an n-value meta tensor (group 0: one group)."""
    if n == 0:
        return 0
    return 1 if group == 0 else -(-n // group)


def meta_quantize(x, group: int) -> dict:
    """8-bit min-max round-to-nearest of an fp16 vector (zero points or scales),
    groups of ``group`` consecutive values (ragged last group; 0 = one group).
    Returns uint8 codes and the fp16 scale and zero of every group."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float16).reshape(-1)
    ng = meta_groups(x.size, group)
    codes = np.empty(x.size, np.uint8)
    scale = np.empty(ng, np.uint16)
    zero = np.empty(ng, np.uint16)
    st = lib.hqq_oracle_meta_quantize(_ptr(x.view(np.uint16)), x.size, group, _ptr(codes),
                                      _ptr(scale), _ptr(zero))
    if st:
        raise ValueError(f"meta_quantize rejected the arguments (status {st})")
    return dict(codes=codes, scale=scale.view(np.float16), zero=zero.view(np.float16))


def meta_dequantize(codes, scale, zero, group: int) -> np.ndarray:
    """fp16((c - z) * s) of 8-bit meta codes with their groups' fp16 s and z."""
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8).reshape(-1)
    scale = np.ascontiguousarray(scale, dtype=np.float16).reshape(-1)
    zero = np.ascontiguousarray(zero, dtype=np.float16).reshape(-1)
    out = np.empty(codes.size, np.uint16)
    st = lib.hqq_oracle_meta_dequantize(_ptr(codes), _ptr(scale.view(np.uint16)),
                                        _ptr(zero.view(np.uint16)), codes.size, group,
                                        _ptr(out))
    if st:
        raise ValueError(f"meta_dequantize rejected the arguments (status {st})")
    return out.view(np.float16)


def dequantize_meta(codes, group: int, zero_q: dict, zero_group: int = 0,
                    scale=None, scale_q: dict | None = None,
                    scale_group: int = 128) -> np.ndarray:
    """Weights from codes whose zero points (and optionally scales) are stored
    8-bit: the zero points and scales are first restored to fp16 by
    ``meta_dequantize``, then ``dequantize`` runs as usual.  Exactly one of
    ``scale`` (fp16 per group) and ``scale_q`` (a ``meta_quantize`` result) is
    given."""
    z = meta_dequantize(zero_q["codes"], zero_q["scale"], zero_q["zero"], zero_group)
    if (scale is None) == (scale_q is None):
        raise ValueError("give exactly one of scale and scale_q")
    s = scale if scale_q is None else meta_dequantize(
        scale_q["codes"], scale_q["scale"], scale_q["zero"], scale_group)
    return dequantize(codes, s, z, group)


def linear(X, W_hat) -> dict:
    """Weight-only linear layer on dequantized weights: Y = X W_hat^T.

    X is fp16 [M, K] (tokens x input features), W_hat the fp16 [N, K] matrix
    that ``dequantize`` restores (output x input features).  The products and
    their sum are formed in fp64 (numpy matmul), then rounded once to fp16.
    Returns the fp16 result, the fp64 result and sum_k |x||w| per output (the
    scale of the rounding bound of any binary32 summation order)."""
    X64 = np.asarray(X, dtype=np.float16).astype(np.float64)
    W64 = np.asarray(W_hat, dtype=np.float16).astype(np.float64)
    Y64 = X64 @ W64.T
    absum = np.abs(X64) @ np.abs(W64).T
    return dict(y=Y64.astype(np.float16), y64=Y64, absum=absum)


def quant_error(W, codes, scale, zero, group: int) -> np.ndarray:
    """Delta W = W - W_hat in fp64 (exact: both are fp16), W_hat from ``dequantize``."""
    W64 = np.asarray(W, dtype=np.float16).astype(np.float64)
    Wh = dequantize(codes, scale, zero, group).astype(np.float64).reshape(W64.shape)
    return W64 - Wh


def lowrank(dW, rank: int) -> dict:
    """Rank-r residual of the quantization error by plain SVD ("Boost 2-bit LLM
    accuracy with EoRA", the section on finding adapters in the feature space:
    Delta W = U Sigma V^T, B = U_r Sigma_r, A = V_r^T; the Eckart-Young optimum
    in the Frobenius norm).  Library SVD in fp64 on the exact Delta W.

    Returns B [N, r], A [r, K], the r leading singular values and all of them.
    The factors are unique up to the signs of matching columns of B and rows of
    A when sigma_r > sigma_{r+1}; B @ A is then unique."""
    dW = np.asarray(dW, dtype=np.float64)
    U, S, Vt = np.linalg.svd(dW, full_matrices=False)
    return dict(B=U[:, :rank] * S[:rank], A=Vt[:rank].copy(), sigma=S[:rank].copy(), sigma_all=S)


def f32_to_f16(x) -> np.ndarray:
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.size, np.uint16)
    lib.hqq_oracle_f32_to_f16(_ptr(x), x.size, _ptr(out))
    return out.view(np.float16).reshape(x.shape)


def lp_error(W, W_hat, p: float = 0.7) -> float:
    """Per-tensor sum |W - W_hat|^p in fp64 (the parity metric; plain numpy)."""
    a = np.asarray(W, dtype=np.float64).reshape(-1)
    b = np.asarray(W_hat, dtype=np.float64).reshape(-1)
    return float(np.sum(np.abs(a - b) ** p))
