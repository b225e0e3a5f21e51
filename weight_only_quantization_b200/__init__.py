"""Python binding of libhqq (include/hqq.h): HQQ group-wise weight-only
quantization of fp16 weight matrices on NVIDIA B200 (sm_100a).

Argument marshalling only: every step of the quantization and dequantization
runs in libhqq's CUDA kernels.  torch supplies device memory and the current
stream.  There is no fallback: importing fails loudly when libhqq.so is absent,
and every call raises ``HQQError`` on a non-zero status.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

__all__ = ["HQQError", "hqq_quantize", "hqq_quantize_ex", "hqq_quantize_half", "hqq_dequantize",
           "hqq_packed_bytes", "hqq_status_string", "QuantizedMatrix", "LIB_PATH",
           "Meta8", "hqq_meta_groups", "hqq_meta_quantize", "hqq_meta_quantize_batch",
           "hqq_meta_dequantize",
           "hqq_dequantize_meta", "hqq_linear", "hqq_linear_meta",
           "DEFAULT_P", "DEFAULT_BETA", "DEFAULT_KAPPA", "DEFAULT_ITERS"]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhqq.so")

DEFAULT_P, DEFAULT_BETA, DEFAULT_KAPPA, DEFAULT_ITERS = 0.7, 1.0, 1.01, 20

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python weight_only_quantization_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)
_P, _I64, _I, _F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
_lib.hqq_packed_bytes.argtypes = [_I64, _I64, _I]
_lib.hqq_packed_bytes.restype = _I64
_lib.hqq_status_string.argtypes = [_I]
_lib.hqq_status_string.restype = ctypes.c_char_p
_lib.hqq_quantize.argtypes = [_P, _I64, _I64, _I, _I, _F, _F, _F, _I, _P, _P, _P, _P]
_lib.hqq_quantize.restype = _I
_lib.hqq_quantize_ex.argtypes = [_P, _I64, _I64, _I, _I, _F, _F, _F, _I, _P, _P, _P, _P, _P, _P,
                                 _P]
_lib.hqq_quantize_ex.restype = _I
_lib.hqq_quantize_half.argtypes = [_P, _I64, _I64, _I, _I, _F, _F, _F, _I, _P, _P, _P, _P, _P, _P,
                                   _P, _P]
_lib.hqq_quantize_half.restype = _I
_lib.hqq_dequantize.argtypes = [_P, _P, _P, _I64, _I64, _I, _I, _P, _P]
_lib.hqq_dequantize.restype = _I
_lib.hqq_meta_groups.argtypes = [_I64, _I64]
_lib.hqq_meta_groups.restype = _I64
_lib.hqq_meta_quantize.argtypes = [_P, _I64, _I64, _P, _P, _P, _P]
_lib.hqq_meta_quantize.restype = _I
_lib.hqq_meta_dequantize.argtypes = [_P, _P, _P, _I64, _I64, _P, _P]
_lib.hqq_meta_dequantize.restype = _I


class _CMeta8(ctypes.Structure):
    """struct hqq_meta8 of include/hqq.h."""
    _fields_ = [("codes", _P), ("scale", _P), ("zero", _P), ("group", _I64)]


class _CMetaJob(ctypes.Structure):
    """struct hqq_meta_job of include/hqq.h."""
    _fields_ = [("x", _P), ("n", _I64), ("mgroup", _I64), ("codes", _P), ("scale", _P),
                ("zero", _P)]


_lib.hqq_meta_quantize_batch.argtypes = [ctypes.POINTER(_CMetaJob), _I64, _P]
_lib.hqq_meta_quantize_batch.restype = _I
_lib.hqq_dequantize_meta.argtypes = [_P, ctypes.POINTER(_CMeta8), _P, ctypes.POINTER(_CMeta8),
                                     _I64, _I64, _I, _I, _P, _P]
_lib.hqq_dequantize_meta.restype = _I
_lib.hqq_linear.argtypes = [_P, _I64, _P, _P, _P, _I64, _I64, _I, _I, _P, _P, _P]
_lib.hqq_linear.restype = _I
_lib.hqq_linear_meta.argtypes = [_P, _I64, _P, ctypes.POINTER(_CMeta8), _P,
                                 ctypes.POINTER(_CMeta8), _I64, _I64, _I, _I, _P, _P, _P]
_lib.hqq_linear_meta.restype = _I
_lib.hqq_lowrank_workspace_bytes.argtypes = [_I64, _I64, _I]
_lib.hqq_lowrank_workspace_bytes.restype = _I64
_lib.hqq_lowrank.argtypes = [_P, _P, _P, _P, _I64, _I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                             _I64, _P]
_lib.hqq_lowrank.restype = _I


class HQQError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        super().__init__(hqq_status_string(status))


def hqq_status_string(status: int) -> str:
    return _lib.hqq_status_string(status).decode()


def hqq_packed_bytes(rows: int, cols: int, nbits: int) -> int:
    n = _lib.hqq_packed_bytes(rows, cols, nbits)
    if n < 0:
        raise HQQError(2 if nbits in (1, 2, 3, 4, 8) else 3)
    return int(n)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st: int):
    if st != 0:
        raise HQQError(st)


@dataclass
class QuantizedMatrix:
    """Packed codes + fp16 scale/zero of one [rows, cols] matrix."""
    packed: "torch.Tensor"     # uint8 [hqq_packed_bytes]
    scale: "torch.Tensor"      # fp16 [rows, cols/group]
    zero: "torch.Tensor"       # fp16 [rows, cols/group]
    rows: int
    cols: int
    nbits: int
    group: int
    zero_f32: "torch.Tensor | None" = None
    iters: "torch.Tensor | None" = None
    err: "torch.Tensor | None" = None
    half: "torch.Tensor | None" = None      # uint8: group solved in half precision


def _outputs(W, nbits, group, packed, scale, zero):
    import torch
    rows, cols = W.shape
    if packed is None:
        packed = torch.empty(hqq_packed_bytes(rows, cols, nbits), dtype=torch.uint8,
                             device=W.device)
    meta = (rows, cols // group if group > 0 else 0)
    if scale is None:
        scale = torch.empty(meta, dtype=torch.float16, device=W.device)
    if zero is None:
        zero = torch.empty(meta, dtype=torch.float16, device=W.device)
    return packed, scale, zero


def _check_tensor(t, name):
    if t is not None and not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def _precision(precision: str) -> bool:
    if precision not in ("fp32", "fp16"):
        raise ValueError("precision must be 'fp32' (single-precision solver) or 'fp16' "
                         "(the half-precision solver)")
    return precision == "fp16"


def hqq_quantize(W, nbits: int = 4, group: int = 64, p: float = DEFAULT_P,
                 beta: float = DEFAULT_BETA, kappa: float = DEFAULT_KAPPA,
                 iters: int = DEFAULT_ITERS, packed=None, scale=None, zero=None,
                 stream=None, precision: str = "fp32") -> QuantizedMatrix:
    """Quantize a contiguous fp16 CUDA matrix [rows, cols] (see include/hqq.h);
    ``precision="fp16"`` runs the half-precision solver (hqq_quantize_half)."""
    import torch
    if W.dtype != torch.float16 or W.dim() != 2:
        raise ValueError("W must be a 2-D float16 tensor")
    half = _precision(precision)
    for t, n in ((W, "W"), (packed, "packed"), (scale, "scale"), (zero, "zero")):
        _check_tensor(t, n)
    packed, scale, zero = _outputs(W, nbits, group, packed, scale, zero)
    rows, cols = W.shape
    if half:
        _check(_lib.hqq_quantize_half(_ptr(W), rows, cols, nbits, group, p, beta, kappa, iters,
                                      _ptr(packed), _ptr(scale), _ptr(zero), None, None, None,
                                      None, _stream(stream)))
    else:
        _check(_lib.hqq_quantize(_ptr(W), rows, cols, nbits, group, p, beta, kappa, iters,
                                 _ptr(packed), _ptr(scale), _ptr(zero), _stream(stream)))
    return QuantizedMatrix(packed, scale, zero, rows, cols, nbits, group)


def hqq_quantize_ex(W, nbits: int = 4, group: int = 64, p: float = DEFAULT_P,
                    beta: float = DEFAULT_BETA, kappa: float = DEFAULT_KAPPA,
                    iters: int = DEFAULT_ITERS, packed=None, scale=None, zero=None,
                    zero_f32=None, iters_out=None, err_out=None, stream=None,
                    precision: str = "fp32", half_out=None) -> QuantizedMatrix:
    """hqq_quantize plus the fp32 zero, the solver's l_p error and the
    accepted-iteration count of every group (and, with ``precision="fp16"``,
    which groups were solved in half precision)."""
    import torch
    if W.dtype != torch.float16 or W.dim() != 2:
        raise ValueError("W must be a 2-D float16 tensor")
    half = _precision(precision)
    for t, n in ((W, "W"), (packed, "packed"), (scale, "scale"), (zero, "zero"),
                 (zero_f32, "zero_f32"), (iters_out, "iters_out"), (err_out, "err_out")):
        _check_tensor(t, n)
    packed, scale, zero = _outputs(W, nbits, group, packed, scale, zero)
    rows, cols = W.shape
    meta = (rows, cols // group if group > 0 else 0)
    if zero_f32 is None:
        zero_f32 = torch.empty(meta, dtype=torch.float32, device=W.device)
    if iters_out is None:
        iters_out = torch.empty(meta, dtype=torch.uint8, device=W.device)
    if err_out is None:
        err_out = torch.empty(meta, dtype=torch.float32, device=W.device)
    if half:
        _check_tensor(half_out, "half_out")
        if half_out is None:
            half_out = torch.empty(meta, dtype=torch.uint8, device=W.device)
        _check(_lib.hqq_quantize_half(_ptr(W), rows, cols, nbits, group, p, beta, kappa, iters,
                                      _ptr(packed), _ptr(scale), _ptr(zero), _ptr(zero_f32),
                                      _ptr(err_out), _ptr(iters_out), _ptr(half_out),
                                      _stream(stream)))
    else:
        half_out = None
        _check(_lib.hqq_quantize_ex(_ptr(W), rows, cols, nbits, group, p, beta, kappa, iters,
                                    _ptr(packed), _ptr(scale), _ptr(zero), _ptr(zero_f32),
                                    _ptr(err_out), _ptr(iters_out), _stream(stream)))
    return QuantizedMatrix(packed, scale, zero, rows, cols, nbits, group, zero_f32, iters_out,
                           err_out, half_out)


def hqq_dequantize(q: QuantizedMatrix, out=None, stream=None):
    """fp16 [rows, cols] = (code - zero) * scale  (see include/hqq.h)."""
    import torch
    for t, n in ((q.packed, "packed"), (q.scale, "scale"), (q.zero, "zero"), (out, "out")):
        _check_tensor(t, n)
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=torch.float16, device=q.packed.device)
    _check(_lib.hqq_dequantize(_ptr(q.packed), _ptr(q.scale), _ptr(q.zero), q.rows, q.cols,
                               q.nbits, q.group, _ptr(out), _stream(stream)))
    return out


@dataclass
class Meta8:
    """8-bit form of a meta tensor (a matrix's zero points or scales)."""
    codes: "torch.Tensor"      # uint8 [n]
    scale: "torch.Tensor"      # fp16 [hqq_meta_groups(n, group)]
    zero: "torch.Tensor"       # fp16 [hqq_meta_groups(n, group)]
    group: int                 # 0 (one group) or a power of two

    def _c(self):
        return _CMeta8(self.codes.data_ptr(), self.scale.data_ptr(), self.zero.data_ptr(),
                       self.group)


def hqq_meta_groups(n: int, mgroup: int) -> int:
    g = _lib.hqq_meta_groups(n, mgroup)
    if g < 0:
        raise HQQError(2)
    return int(g)


def hqq_meta_quantize(x, mgroup: int = 0, codes=None, scale=None, zero=None,
                      stream=None) -> Meta8:
    """8-bit min-max round-to-nearest of an fp16 meta tensor (flat order;
    ``mgroup`` consecutive values per group, 0 = one group); see include/hqq.h."""
    import torch
    if x.dtype != torch.float16:
        raise ValueError("x must be float16")
    _check_tensor(x, "x")
    n = x.numel()
    ng = hqq_meta_groups(n, mgroup)
    if codes is None:
        codes = torch.empty(n, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(ng, dtype=torch.float16, device=x.device)
    if zero is None:
        zero = torch.empty(ng, dtype=torch.float16, device=x.device)
    for t, nm in ((codes, "codes"), (scale, "scale"), (zero, "zero")):
        _check_tensor(t, nm)
    _check(_lib.hqq_meta_quantize(_ptr(x), n, mgroup, _ptr(codes), _ptr(scale), _ptr(zero),
                                  _stream(stream)))
    return Meta8(codes, scale, zero, mgroup)


def hqq_meta_quantize_batch(tensors, stream=None, outputs=None) -> list:
    """hqq_meta_quantize of many fp16 meta tensors in shared launches.
    ``tensors`` is a list of (x, mgroup); ``outputs`` optionally a list of
    Meta8 to write into (same order).  Returns the list of Meta8."""
    import torch
    out = []
    jobs = (_CMetaJob * max(len(tensors), 1))()
    for i, (x, mgroup) in enumerate(tensors):
        if x.dtype != torch.float16:
            raise ValueError("x must be float16")
        _check_tensor(x, "x")
        n = x.numel()
        if outputs is not None:
            m = outputs[i]
        else:
            ng = hqq_meta_groups(n, mgroup)
            m = Meta8(torch.empty(n, dtype=torch.uint8, device=x.device),
                      torch.empty(ng, dtype=torch.float16, device=x.device),
                      torch.empty(ng, dtype=torch.float16, device=x.device), mgroup)
        for t, nm in ((m.codes, "codes"), (m.scale, "scale"), (m.zero, "zero")):
            _check_tensor(t, nm)
        jobs[i] = _CMetaJob(x.data_ptr(), n, mgroup, m.codes.data_ptr(), m.scale.data_ptr(),
                            m.zero.data_ptr())
        out.append(m)
    _check(_lib.hqq_meta_quantize_batch(jobs, len(tensors), _stream(stream)))
    return out


def hqq_meta_dequantize(m: Meta8, out=None, stream=None):
    """fp16 [n] = (code - zero) * scale per value of an 8-bit meta tensor."""
    import torch
    for t, nm in ((m.codes, "codes"), (m.scale, "scale"), (m.zero, "zero"), (out, "out")):
        _check_tensor(t, nm)
    n = m.codes.numel()
    if out is None:
        out = torch.empty(n, dtype=torch.float16, device=m.codes.device)
    _check(_lib.hqq_meta_dequantize(_ptr(m.codes), _ptr(m.scale), _ptr(m.zero), n, m.group,
                                    _ptr(out), _stream(stream)))
    return out


def hqq_dequantize_meta(packed, zero_q: Meta8, rows: int, cols: int, nbits: int, group: int,
                        scale=None, scale_q: Meta8 | None = None, out=None, stream=None):
    """Dequantize a matrix whose zero points (and optionally scales) are kept in
    8-bit form, in one pass (see include/hqq.h)."""
    import torch
    for t, nm in ((packed, "packed"), (scale, "scale"), (out, "out")):
        _check_tensor(t, nm)
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float16, device=packed.device)
    zc = zero_q._c()
    sc = scale_q._c() if scale_q is not None else None
    _check(_lib.hqq_dequantize_meta(_ptr(packed), ctypes.byref(zc), _ptr(scale),
                                    ctypes.byref(sc) if sc is not None else None,
                                    rows, cols, nbits, group, _ptr(out), _stream(stream)))
    return out


def hqq_linear(X, q: QuantizedMatrix, out=None, status=None, stream=None):
    """Y = X W_hat^T for fp16 X [M, cols] and a quantized [rows, cols] matrix,
    with the dequantization fused into the tensor-core product (see
    include/hqq.h).  ``status`` is an optional int32 CUDA tensor of one element
    (cleared by the caller) that the kernel sets to 1 if an internal wait ran
    out."""
    import torch
    if X.dtype != torch.float16 or X.dim() != 2 or X.shape[1] != q.cols:
        raise ValueError("X must be a float16 [M, cols] tensor")
    for t, nm in ((X, "X"), (q.packed, "packed"), (q.scale, "scale"), (q.zero, "zero"),
                  (out, "out"), (status, "status")):
        _check_tensor(t, nm)
    if out is None:
        out = torch.empty((X.shape[0], q.rows), dtype=torch.float16, device=X.device)
    _check(_lib.hqq_linear(_ptr(X), X.shape[0], _ptr(q.packed), _ptr(q.scale), _ptr(q.zero),
                           q.rows, q.cols, q.nbits, q.group, _ptr(out), _ptr(status),
                           _stream(stream)))
    return out


def hqq_linear_meta(X, packed, zero_q: Meta8, rows: int, cols: int, nbits: int, group: int,
                    scale=None, scale_q: Meta8 | None = None, out=None, status=None,
                    stream=None):
    """hqq_linear for a matrix whose zero points (and optionally scales) are
    kept in 8-bit form; they are restored inside the kernel (see include/hqq.h)."""
    import torch
    if X.dtype != torch.float16 or X.dim() != 2 or X.shape[1] != cols:
        raise ValueError("X must be a float16 [M, cols] tensor")
    for t, nm in ((X, "X"), (packed, "packed"), (scale, "scale"), (out, "out"),
                  (status, "status")):
        _check_tensor(t, nm)
    if out is None:
        out = torch.empty((X.shape[0], rows), dtype=torch.float16, device=X.device)
    zc = zero_q._c()
    sc = scale_q._c() if scale_q is not None else None
    _check(_lib.hqq_linear_meta(_ptr(X), X.shape[0], _ptr(packed), ctypes.byref(zc),
                                _ptr(scale), ctypes.byref(sc) if sc is not None else None,
                                rows, cols, nbits, group, _ptr(out), _ptr(status),
                                _stream(stream)))
    return out


def hqq_lowrank(W, q: QuantizedMatrix, rank: int, omega, power_iters: int = 2, workspace=None,
                stream=None):
    """Rank-r residual B [rows, rank], A [rank, cols] (fp32) of the quantization
    error W - W_hat, with the r leading singular values (see include/hqq.h).
    ``omega`` is the fp32 [cols, sketch] Gaussian test matrix (sketch 16, 32 or
    64), drawn by the caller; the workspace is allocated here unless given."""
    import torch
    if W.dtype != torch.float16 or tuple(W.shape) != (q.rows, q.cols):
        raise ValueError("W must be the float16 [rows, cols] matrix that q quantizes")
    if omega.dtype != torch.float32 or omega.dim() != 2 or omega.shape[0] != q.cols:
        raise ValueError("omega must be a float32 [cols, sketch] tensor")
    for t, nm in ((W, "W"), (omega, "omega"), (workspace, "workspace")):
        _check_tensor(t, nm)
    sketch = omega.shape[1]
    need = _lib.hqq_lowrank_workspace_bytes(q.rows, q.cols, sketch)
    if need < 0:
        raise ValueError("sketch must be 16, 32 or 64")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    B = torch.empty((q.rows, rank), dtype=torch.float32, device=W.device)
    A = torch.empty((rank, q.cols), dtype=torch.float32, device=W.device)
    sigma = torch.empty(rank, dtype=torch.float32, device=W.device)
    _check(_lib.hqq_lowrank(_ptr(W), _ptr(q.packed), _ptr(q.scale), _ptr(q.zero), q.rows, q.cols,
                            q.nbits, q.group, rank, sketch, power_iters, _ptr(omega), _ptr(B),
                            _ptr(A), _ptr(sigma), _ptr(workspace), workspace.numel(),
                            _stream(stream)))
    return B, A, sigma
