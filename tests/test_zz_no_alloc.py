"""hqq_lowrank_noalloc: the low-rank residual for callers that cannot allocate
device memory (code running where cudaMalloc is unavailable or forbidden, such
as a plugin inside a framework that owns the allocator).  It runs the same
kernels as hqq_lowrank on a fixed scratch array inside the library, so through
the C ABI it must give hqq_lowrank's results (within the low-rank tests'
tolerance) on two calls in a row, the second reusing the scratch that the first
left behind, and must turn away a matrix whose workspace exceeds that array.

This file is collected last on purpose: the entry point keeps process-wide
state (the per-device scratch address), and a failure here should come after
every other test has run."""
import ctypes

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

_P, _I, _I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_the_workspace_entry_point():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import weight_only_quantization_b200 as hqq
    lib = hqq._lib
    fn = lib.hqq_lowrank_noalloc
    fn.argtypes = [_P, _P, _P, _P, _I64, _I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P]
    fn.restype = _I
    lib.hqq_lowrank_noalloc_max_bytes.argtypes = []
    lib.hqq_lowrank_noalloc_max_bytes.restype = _I64
    assert lib.hqq_lowrank_noalloc_max_bytes() == 16 << 20
    for rows, cols, nbits, group, rank, sketch, seed in [(512, 1024, 3, 64, 16, 32, 1),
                                                         (384, 256, 4, 32, 8, 16, 2)]:
        W = synth.student_t_device((rows, cols), seed=80, stream=seed)
        q = hqq.hqq_quantize(W, nbits=nbits, group=group)
        rng = np.random.default_rng(seed)
        om = torch.from_numpy(rng.standard_normal((cols, sketch)).astype(np.float32)).cuda()
        Bw, Aw, sw = hqq.hqq_lowrank(W, q, rank, om, power_iters=2)
        ref = (Bw.double() @ Aw.double())
        for _ in range(2):
            B = torch.full((rows, rank), float("nan"), device="cuda")
            A = torch.full((rank, cols), float("nan"), device="cuda")
            s = torch.full((rank,), float("nan"), device="cuda")
            st = fn(_ptr(W), _ptr(q.packed), _ptr(q.scale), _ptr(q.zero), rows, cols, nbits,
                    group, rank, sketch, 2, _ptr(om), _ptr(B), _ptr(A), _ptr(s), None)
            assert st == 0, hqq.status_string(st) if hasattr(hqq, "status_string") else st
            torch.cuda.synchronize()
            assert float((s.double() - sw.double()).abs().max()) <= 1e-4 * float(sw[0])
            got = B.double() @ A.double()
            assert float((got - ref).abs().max()) <= 1e-4 * float(ref.abs().max())
    # a workspace beyond the fixed array is turned away before anything runs
    assert lib.hqq_lowrank_workspace_bytes(65536, 8192, 64) > 16 << 20
    st = fn(_P(256), _P(256), _P(256), _P(256), 65536, 8192, 4, 64, 8, 64, 2, _P(256), _P(256),
            _P(256), None, None)
    assert st == 7
