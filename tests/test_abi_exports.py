"""The C ABI library loads on a machine without a GPU, exports every entry point
declared in include/hqq.h, and rejects bad arguments on the host before any
CUDA call.  No compute call is made here."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hqq.h")


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "hqq_build", os.path.join(ROOT, "weight_only_quantization_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import weight_only_quantization_b200 as hqq
    return hqq


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hqq_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ["hqq_quantize", "hqq_quantize_ex", "hqq_dequantize", "hqq_packed_bytes",
                 "hqq_status_string"]:
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (hqq_\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib._lib, name)


def test_header_compiles_as_c():
    src = '#include "hqq.h"\nint main(void){return (int)hqq_packed_bytes(1,16,4);}\n'
    res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-x", "c",
                          "-I", os.path.join(ROOT, "include"), "-"], input=src, text=True,
                         capture_output=True)
    assert res.returncode == 0, res.stderr


def test_packed_bytes(lib):
    assert lib.hqq_packed_bytes(4096, 4096, 4) == 4096 * 4096 // 2
    assert lib.hqq_packed_bytes(4096, 4096, 2) == 4096 * 4096 // 4
    assert lib.hqq_packed_bytes(4096, 4096, 3) == 4 * ((4096 * 4096 + 9) // 10)
    assert lib.hqq_packed_bytes(1, 64, 3) == 28
    assert lib._lib.hqq_packed_bytes(-1, 64, 4) == -1
    assert lib._lib.hqq_packed_bytes(4, 64, 5) == -1
    assert lib.hqq_packed_bytes(4096, 4096, 8) == 4096 * 4096
    assert lib.hqq_packed_bytes(3, 7, 1) == 3
    assert lib.hqq_packed_bytes(4096, 4096, 1) == 4096 * 4096 // 8


def test_status_strings(lib):
    for s in range(7):
        assert lib.hqq_status_string(s).startswith("HQQ_")
    assert "unknown" in lib.hqq_status_string(99)


def test_host_validation_without_gpu(lib):
    L = lib._lib
    P = lambda v: ctypes.c_void_p(v)
    a = dict(rows=64, cols=256, nbits=4, group=64, p=0.7, beta=1.0, kappa=1.01, iters=20)
    cases = [
        (dict(nbits=5), 3), (dict(nbits=0), 3), (dict(nbits=6), 3), (dict(group=48), 3), (dict(group=8), 3),
        (dict(group=512), 3), (dict(cols=250), 2), (dict(rows=-3), 2),
        (dict(p=0.0), 4), (dict(p=1.0001), 4), (dict(p=float("nan")), 4),
        (dict(beta=0.0), 4), (dict(beta=float("inf")), 4), (dict(kappa=0.0), 4),
        (dict(kappa=float("nan")), 4), (dict(iters=-1), 4), (dict(iters=256), 4),
    ]
    for over, want in cases:
        b = dict(a, **over)
        st = L.hqq_quantize(P(256), b["rows"], b["cols"], b["nbits"], b["group"], b["p"],
                            b["beta"], b["kappa"], b["iters"], P(256), P(256), P(256), None)
        assert st == want, (over, st)
    # null and misaligned pointers
    assert L.hqq_quantize(None, 64, 256, 4, 64, 0.7, 1.0, 1.01, 20, P(256), P(256), P(256),
                          None) == 1
    assert L.hqq_quantize(P(258), 64, 256, 4, 64, 0.7, 1.0, 1.01, 20, P(256), P(256), P(256),
                          None) == 5
    assert L.hqq_quantize(P(256), 64, 256, 4, 64, 0.7, 1.0, 1.01, 20, P(258), P(256), P(256),
                          None) == 5
    assert L.hqq_quantize_ex(P(256), 64, 256, 4, 64, 0.7, 1.0, 1.01, 20, P(256), P(256),
                             P(256), P(258), None, None, None) == 5
    assert L.hqq_quantize_ex(P(256), 64, 256, 4, 64, 0.7, 1.0, 1.01, 20, P(256), P(256),
                             P(256), None, P(262), None, None) == 5
    # empty matrices are valid no-ops (nothing launched, so no GPU needed)
    assert L.hqq_quantize(None, 0, 256, 4, 64, 0.7, 1.0, 1.01, 20, None, None, None, None) == 0
    assert L.hqq_dequantize(None, None, None, 16, 0, 3, 64, None, None) == 0
    # dequantize validation
    assert L.hqq_dequantize(P(256), P(256), P(256), 64, 256, 6, 64, P(256), None) == 3
    assert L.hqq_dequantize(P(256), P(256), None, 64, 256, 4, 64, P(256), None) == 1
    assert L.hqq_dequantize(P(256), P(256), P(256), 64, 256, 4, 64, P(264), None) == 5
    assert L.hqq_dequantize(P(256), P(256), P(256), 64, 100, 4, 64, P(256), None) == 2


def test_meta_host_validation_without_gpu(lib):
    L = lib._lib
    P = lambda v: ctypes.c_void_p(v)
    assert lib.hqq_meta_groups(0, 128) == 0
    assert lib.hqq_meta_groups(1000, 0) == 1
    assert lib.hqq_meta_groups(1000, 128) == 8
    assert L.hqq_meta_groups(-1, 0) == -1
    # quantize: shape, group, null, alignment; n == 0 is a no-op
    assert L.hqq_meta_quantize(P(256), -1, 0, P(256), P(256), P(256), None) == 2
    assert L.hqq_meta_quantize(P(256), 100, 100, P(256), P(256), P(256), None) == 3
    assert L.hqq_meta_quantize(P(256), 100, 1 << 31, P(256), P(256), P(256), None) == 3
    assert L.hqq_meta_quantize(None, 100, 0, P(256), P(256), P(256), None) == 1
    assert L.hqq_meta_quantize(P(258), 100, 0, P(256), P(256), P(256), None) == 5
    assert L.hqq_meta_quantize(P(256), 100, 0, P(260), P(256), P(256), None) == 5
    assert L.hqq_meta_quantize(P(256), 100, 128, P(256), P(257), P(256), None) == 5
    assert L.hqq_meta_quantize(None, 0, 0, None, None, None, None) == 0
    # dequantize
    assert L.hqq_meta_dequantize(P(256), P(256), P(256), 100, 3, P(256), None) == 3
    assert L.hqq_meta_dequantize(P(256), None, P(256), 100, 0, P(256), None) == 1
    assert L.hqq_meta_dequantize(P(256), P(256), P(256), 100, 0, P(264), None) == 5
    assert L.hqq_meta_dequantize(None, None, None, 0, 0, None, None) == 0
    # fused weight dequantize with 8-bit meta data
    M = lib._CMeta8
    good = M(256, 256, 256, 0)
    bad_group = M(256, 256, 256, 96)
    no_codes = M(None, 256, 256, 0)
    r = ctypes.byref
    assert L.hqq_dequantize_meta(P(256), r(good), P(256), r(good), 64, 256, 4, 64, P(256),
                                 None) == 4
    assert L.hqq_dequantize_meta(P(256), r(good), None, None, 64, 256, 4, 64, P(256), None) == 1
    assert L.hqq_dequantize_meta(P(256), None, P(256), None, 64, 256, 4, 64, P(256), None) == 1
    assert L.hqq_dequantize_meta(P(256), r(no_codes), P(256), None, 64, 256, 4, 64, P(256),
                                 None) == 1
    assert L.hqq_dequantize_meta(P(256), r(bad_group), P(256), None, 64, 256, 4, 64, P(256),
                                 None) == 3
    assert L.hqq_dequantize_meta(P(256), r(good), P(256), None, 64, 256, 4, 64, P(260),
                                 None) == 5
    assert L.hqq_dequantize_meta(P(256), r(good), P(256), None, 64, 256, 5, 64, P(256),
                                 None) == 3
    assert L.hqq_dequantize_meta(None, None, None, None, 0, 256, 4, 64, None, None) == 0
    # linear layer with 8-bit meta data: argument checks before any launch
    assert L.hqq_linear_meta(P(256), 4, P(256), r(good), P(256), r(good), 64, 256, 4, 64,
                             P(256), None, None) == 4
    assert L.hqq_linear_meta(P(256), 4, P(256), None, P(256), None, 64, 256, 4, 64, P(256),
                             None, None) == 1
    assert L.hqq_linear_meta(P(256), 4, P(256), r(bad_group), P(256), None, 64, 256, 4, 64,
                             P(256), None, None) == 3
    assert L.hqq_linear_meta(P(264), 4, P(256), r(good), P(256), None, 64, 256, 4, 64,
                             P(256), None, None) == 5
    assert L.hqq_linear_meta(None, 0, None, None, None, None, 64, 256, 4, 64, None, None,
                             None) == 0


def test_lowrank_host_validation_without_gpu(lib):
    L = lib._lib
    P = lambda v: ctypes.c_void_p(v)
    ws = L.hqq_lowrank_workspace_bytes(256, 512, 32)
    assert ws > 0 and ws % 256 == 0
    assert L.hqq_lowrank_workspace_bytes(256, 512, 24) == -1
    assert L.hqq_lowrank_workspace_bytes(-1, 512, 32) == -1
    assert L.hqq_lowrank_workspace_bytes(256, 512, 64) > ws

    def call(rows=256, cols=512, nbits=4, group=64, rank=8, sketch=32, iters=2, omega=256,
             W=256, B=256, A=256, sigma=None, wsp=256, wsb=ws):
        if wsb == ws:
            wsb = L.hqq_lowrank_workspace_bytes(max(rows, 0), max(cols, 0), sketch) \
                if sketch in (16, 32, 64) and rows >= 0 and cols >= 0 else ws
        return L.hqq_lowrank(P(W) if W else None, P(256), P(256), P(256), rows, cols, nbits,
                             group, rank, sketch, iters, P(omega) if omega else None,
                             P(B) if B else None, P(A) if A else None,
                             P(sigma) if sigma else None, P(wsp) if wsp else None, wsb, None)
    assert call(sketch=24) == 3
    assert call(nbits=5) == 3
    assert call(rank=0) == 4
    assert call(rank=33) == 4
    assert call(iters=-1) == 4
    assert call(iters=17) == 4
    assert call(rows=16) == 2
    assert call(cols=16, group=16) == 2
    assert call(cols=500) == 2
    assert call(W=0) == 1
    assert call(omega=0) == 1
    assert call(wsp=0) == 1
    assert call(wsb=ws - 1) == 4
    assert call(W=264) == 5
    assert call(omega=260) == 5
    assert call(B=258) == 5
    assert call(sigma=258) == 5
    assert call(wsp=384) == 5
