"""GPU parity: libhqq (through its C ABI) against the CPU oracle, element by
element on the same seeded inputs.  Tolerances are defined in tests/_parity.py.
"""
import numpy as np
import pytest

import oracle
import synth
from _parity import compare_full, gpu_quantize, group_codes, to_np, ZERO_TOL, CODE_MATCH

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def hqq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import weight_only_quantization_b200 as m   # raises if libhqq.so is missing
    return m


def _dev_weights(shape, seed, stream=0, std=synth.STD):
    W = synth.student_t_device(shape, seed=seed, stream=stream, std=std)
    torch.cuda.synchronize()
    return W, W.cpu().numpy()


def _check(hqq, W_dev, W_np, nbits, group, label, **kw):
    gq = to_np(gpu_quantize(W_dev, nbits, group, **kw))
    ref = oracle.quantize(W_np, nbits, group, **kw)
    st = compare_full(W_np, gq, ref, nbits, group, p=kw.get("p", 0.7), label=label)
    return gq, ref, st


# ---------------------------------------------------------------- the configs
def test_c1_1024_4bit_g64(hqq):
    W, Wn = _dev_weights((1024, 1024), seed=0)
    _, _, st = _check(hqq, W, Wn, 4, 64, "1024^2 4b g64")
    assert st["code_match"] == 1.0 and st["max_dz"] == 0.0 and st["iters_equal"] == 1.0


@pytest.mark.parametrize("nbits,group", [(4, 64), (2, 32)])
def test_c2_4096(hqq, nbits, group):
    W, Wn = _dev_weights((4096, 4096), seed=1)
    _, _, st = _check(hqq, W, Wn, nbits, group, f"4096^2 {nbits}b g{group}")
    assert st["code_match"] == 1.0 and st["iters_equal"] == 1.0


# ------------------------------------------------- every width x group, ragged
@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("group", [16, 32, 64, 128, 256])
def test_all_formats_ragged(hqq, nbits, group):
    # 37 rows x 13 groups: not a multiple of a CTA tile nor of 5 groups (3-bit words)
    W, Wn = _dev_weights((37, 13 * group), seed=21, stream=nbits * 1000 + group)
    _, _, st = _check(hqq, W, Wn, nbits, group, f"ragged {nbits}b g{group}")
    assert st["code_match"] == 1.0


@pytest.mark.parametrize("shape", [(1, 64), (1, 128), (3, 64), (1, 640), (5, 192)])
@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
def test_odd_shapes(hqq, shape, nbits):
    W, Wn = _dev_weights(shape, seed=22, stream=shape[0] * 7 + shape[1])
    _check(hqq, W, Wn, nbits, 64, f"shape {shape} {nbits}b")


def test_empty_is_noop(hqq):
    W = torch.empty((0, 64), dtype=torch.float16, device="cuda")
    q = hqq.hqq_quantize(W, 4, 64)
    assert q.packed.numel() == 0 and q.scale.numel() == 0
    W = torch.empty((8, 0), dtype=torch.float16, device="cuda")
    q = hqq.hqq_quantize(W, 3, 64)
    out = hqq.hqq_dequantize(q)
    assert out.shape == (8, 0)


# ------------------------------------------------------------ adversarial groups
def _adversarial(G):
    rng = np.random.default_rng(23)
    rows = []
    rows.append(np.zeros(G))                                     # all zero
    rows.append(np.full(G, 0.0137))                              # constant
    rows.append(np.full(G, -65504.0))                            # constant at the range end
    r = rng.standard_normal(G) * 0.02; r[5] = 30.0; rows.append(r)  # one huge outlier
    rows.append(np.linspace(-1, 1, G))                           # evenly spaced: exact ties
    rows.append(np.arange(G) % 16 / 16.0)                        # exact half-way points
    rows.append((rng.standard_normal(G) * 1e-6))                 # fp16 subnormals
    r = np.full(G, 65504.0); r[::2] = -65504.0; rows.append(r)   # +-max fp16
    rows.append(np.where(np.arange(G) < G // 2, 1e-3, -1e-3))    # two levels
    r = rng.standard_normal(G); rows.append(r)                   # unit scale (shrink on)
    r = rng.standard_normal(G) * 10; rows.append(r)              # large scale
    rows.append(np.full(G, 6e-8))                                # constant subnormal
    r = np.zeros(G); r[1::2] = -0.0; r[::3] = 0.25; rows.append(r)  # signed zeros
    return np.array(rows, np.float64).astype(np.float16)


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("group", [16, 64, 128])
def test_adversarial_groups(hqq, nbits, group):
    Wn = _adversarial(group)
    W = torch.from_numpy(Wn).cuda()
    _check(hqq, W, Wn, nbits, group, f"adversarial {nbits}b g{group}")


# ------------------------------------------------- sp1 active: unit-scale weights
@pytest.mark.parametrize("nbits,group", [(4, 64), (2, 32), (3, 64), (2, 128), (8, 128), (1, 64)])
@pytest.mark.parametrize("std", [1.0, 3.0])
def test_shrink_active(hqq, nbits, group, std):
    W, Wn = _dev_weights((256, 1024), seed=24, stream=group, std=std)
    gq, ref, st = _check(hqq, W, Wn, nbits, group, f"std {std} {nbits}b g{group}")
    assert st["code_match"] == 1.0 and st["iters_equal"] == 1.0


# ------------------------- the 20-warp CTA shape, every group compared in full
@pytest.mark.parametrize("nbits,group", [(3, 64), (2, 32), (4, 64)])
@pytest.mark.parametrize("std", [0.02, 3.0])
def test_wide_ctas_full(hqq, nbits, group, std):
    """4096 x 8192 (13108 chunks of 2560 weights): enough chunks that the
    launch takes one 20-warp CTA per SM on a 148-SM B200 rather than two
    8-warp CTAs.  Every group against the oracle, with the shrink inactive
    (std 0.02) and active (std 3), so the clamp and exact-shrink paths of that
    kernel shape run on full-size data."""
    W, Wn = _dev_weights((4096, 8192), seed=25, stream=nbits, std=std)
    _, _, st = _check(hqq, W, Wn, nbits, group, f"wide std {std} {nbits}b g{group}")
    assert st["code_match"] == 1.0 and st["iters_equal"] == 1.0


# ---------------------------------------------------------- solver parameters
@pytest.mark.parametrize("kw", [
    dict(iters=0), dict(iters=1), dict(iters=255), dict(p=1.0), dict(p=0.5),
    dict(p=0.05), dict(beta=0.1), dict(beta=50.0), dict(kappa=1.5), dict(kappa=0.9),
    dict(p=1.0, beta=2.0, kappa=1.2, iters=40),
])
def test_solver_parameters(hqq, kw):
    W, Wn = _dev_weights((128, 1024), seed=25, stream=3, std=0.5)
    gq, ref, st = _check(hqq, W, Wn, 4, 64, f"params {kw}", **kw)
    assert st["code_match"] == 1.0


# ------------------------------------------------------------------ dequantize
@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("group", [16, 32, 64, 128, 256])
def test_dequantize_bitwise(hqq, nbits, group):
    W, Wn = _dev_weights((29, 7 * group), seed=26, stream=group + nbits)
    q = hqq.hqq_quantize(W, nbits, group)
    out = hqq.hqq_dequantize(q)
    torch.cuda.synchronize()
    n = Wn.size
    codes = oracle.unpack(q.packed.cpu().numpy(), n, nbits)
    ref = oracle.dequantize(codes, q.scale.cpu().numpy(), q.zero.cpu().numpy(), group)
    assert np.array_equal(out.cpu().numpy().reshape(-1).view(np.uint16), ref.view(np.uint16))


# ---------------------------------------------- full-size configs, sampled groups
FULL = [
    ("8192x8192 2b g32", (8192, 8192), 2, 32, 3, 0),
    ("8192x8192 2b g128", (8192, 8192), 2, 128, 3, 0),
    ("28672x8192 2b g32", (28672, 8192), 2, 32, 3, 1),
    ("28672x8192 2b g128", (28672, 8192), 2, 128, 3, 1),
    ("70B gate 28672x8192 3b g64", (28672, 8192), 3, 64, 5, 4),
    ("70B down 8192x28672 3b g64", (8192, 28672), 3, 64, 5, 6),
    ("7B up 11008x4096 4b g64", (11008, 4096), 4, 64, 2, 5),
    ("7B down 4096x11008 4b g64", (4096, 11008), 4, 64, 2, 6),
    ("8192x8192 8b g128", (8192, 8192), 8, 128, 7, 0),
    ("8192x8192 1b g64", (8192, 8192), 1, 64, 7, 1),
]


@pytest.mark.parametrize("label,shape,nbits,group,seed,stream", FULL,
                         ids=[f[0] for f in FULL])
def test_full_size_sampled(hqq, label, shape, nbits, group, seed, stream):
    W, _ = None, None
    W = synth.student_t_device(shape, seed=seed, stream=stream)
    q = gpu_quantize(W, nbits, group)
    out = hqq.hqq_dequantize(q)
    torch.cuda.synchronize()
    n_groups = W.numel() // group
    rng = np.random.default_rng(seed * 100 + stream)
    g_idx = np.unique(np.concatenate([rng.integers(0, n_groups, 4000),
                                      [0, 1, n_groups - 1, n_groups - 2]]))
    Wg = W.view(-1, group)[torch.from_numpy(g_idx).cuda()].cpu().numpy()
    ref = oracle.quantize(Wg, nbits, group)
    packed = q.packed.cpu().numpy()
    codes = group_codes(packed, nbits, group, g_idx)
    sc = q.scale.view(-1)[torch.from_numpy(g_idx).cuda()].cpu().numpy()
    zf = q.zero_f32.view(-1)[torch.from_numpy(g_idx).cuda()].cpu().numpy()
    it = q.iters.view(-1)[torch.from_numpy(g_idx).cuda()].cpu().numpy()
    er = q.err.view(-1)[torch.from_numpy(g_idx).cuda()].cpu().numpy()
    assert np.array_equal(er.view(np.uint32), ref["err"].view(np.uint32))
    assert np.array_equal(sc.view(np.uint16), ref["scale"].view(np.uint16))
    assert np.max(np.abs(zf.astype(np.float64) - ref["zero_f32"])) <= ZERO_TOL
    assert np.mean(codes.reshape(-1) == ref["codes"]) >= CODE_MATCH
    assert np.array_equal(it, ref["iters"])
    # dequantized values of the sampled groups against the oracle's Q^-1
    dq = out.view(-1, group)[torch.from_numpy(g_idx).cuda()].cpu().numpy().reshape(-1)
    zq = q.zero.view(-1)[torch.from_numpy(g_idx).cuda()].cpu().numpy()
    dref = oracle.dequantize(codes.reshape(-1), sc, zq, group)
    assert np.array_equal(dq.view(np.uint16), dref.view(np.uint16))
    # 3-bit: the zero padding of the last word
    if nbits == 3 and W.numel() % 10:
        last = int.from_bytes(packed[-4:].tobytes(), "little")
        k = W.numel() % 10
        assert last >> (3 * k) == 0


# --------------------------------------------------------------- ABI behaviour
def test_bad_arguments_touch_nothing(hqq):
    import ctypes
    L = hqq._lib
    W = synth.student_t_device((64, 256), seed=27)
    packed = torch.full((64 * 256 // 2,), 0xAB, dtype=torch.uint8, device="cuda")
    scale = torch.full((64, 4), 7.0, dtype=torch.float16, device="cuda")
    zero = torch.full((64, 4), 7.0, dtype=torch.float16, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [
        (dict(nbits=5), 3), (dict(group=48), 3), (dict(group=512), 3), (dict(cols=250), 2),
        (dict(p=0.0), 4), (dict(p=1.5), 4), (dict(beta=0.0), 4), (dict(kappa=-1.0), 4),
        (dict(iters=256), 4), (dict(iters=-1), 4), (dict(beta=float("inf")), 4),
        (dict(rows=-1), 2),
    ]
    for over, want in cases:
        a = dict(rows=64, cols=256, nbits=4, group=64, p=0.7, beta=1.0, kappa=1.01, iters=20)
        a.update(over)
        st = L.hqq_quantize(P(W), a["rows"], a["cols"], a["nbits"], a["group"], a["p"],
                            a["beta"], a["kappa"], a["iters"], P(packed), P(scale), P(zero), s)
        assert st == want, (over, st)
    assert L.hqq_quantize(None, 64, 256, 4, 64, 0.7, 1.0, 1.01, 20, P(packed), P(scale),
                          P(zero), s) == 1
    misaligned = ctypes.c_void_p(W.data_ptr() + 2)
    assert L.hqq_quantize(misaligned, 64, 256, 4, 64, 0.7, 1.0, 1.01, 20, P(packed), P(scale),
                          P(zero), s) == 5
    torch.cuda.synchronize()
    assert torch.all(packed == 0xAB) and torch.all(scale == 7.0) and torch.all(zero == 7.0)


def test_side_stream_and_no_sync(hqq):
    W, Wn = _dev_weights((512, 1024), seed=28)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        q = hqq.hqq_quantize_ex(W, 3, 64)
        out = hqq.hqq_dequantize(q)
    st.synchronize()
    ref = oracle.quantize(Wn, 3, 64)
    assert np.array_equal(q.scale.cpu().numpy().reshape(-1).view(np.uint16),
                          ref["scale"].view(np.uint16))
    assert np.array_equal(q.packed.cpu().numpy(), ref["packed"])
    dref = oracle.dequantize(ref["codes"], ref["scale"], ref["zero"], 64)
    assert np.array_equal(out.cpu().numpy().reshape(-1).view(np.uint16), dref.view(np.uint16))


def test_repeat_calls_are_deterministic(hqq):
    W, _ = _dev_weights((1024, 4096), seed=29)
    a = hqq.hqq_quantize_ex(W, 4, 64)
    b = hqq.hqq_quantize_ex(W, 4, 64)
    torch.cuda.synchronize()
    assert torch.equal(a.packed, b.packed) and torch.equal(a.zero_f32, b.zero_f32)


# ------------------------------- several chunks per warp (group carry-over path)
@pytest.mark.parametrize("nbits", [8, 4, 3, 2, 1])
@pytest.mark.parametrize("group", [16, 32, 64, 128, 256])
def test_multi_chunk_per_warp(hqq, nbits, group):
    # 16.8 M weights = 6554 chunks of 2560: more than one chunk per resident warp,
    # so groups still running at the end of a chunk are carried to the next one
    W, Wn = _dev_weights((2048, 8192), seed=30, stream=group * 10 + nbits)
    _, _, st = _check(hqq, W, Wn, nbits, group, f"multi-chunk {nbits}b g{group}")
    assert st["code_match"] == 1.0


@pytest.mark.parametrize("group", [64, 16])
def test_multi_chunk_shrink_active(hqq, group):
    W, Wn = _dev_weights((2048, 8192), seed=31, stream=group, std=1.0)
    _check(hqq, W, Wn, 4, group, f"multi-chunk std 1 4b g{group}")


# --------------------------------------- iters = 0: the round-to-nearest kernel
@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("group", [16, 32, 64, 128, 256])
def test_rtn_all_formats_ragged(hqq, nbits, group):
    # 41 rows x 17 groups: several 2560-weight tiles and a ragged last one
    W, Wn = _dev_weights((41, 17 * group), seed=40, stream=nbits * 1000 + group)
    _, _, st = _check(hqq, W, Wn, nbits, group, f"rtn {nbits}b g{group}", iters=0)
    assert st["code_match"] == 1.0


@pytest.mark.parametrize("nbits,group", [(3, 64), (4, 64), (2, 32)])
def test_rtn_full_size_sampled_rows(hqq, nbits, group):
    rows, cols = 28672, 8192
    W = synth.student_t_device((rows, cols), seed=5, stream=4)
    q = gpu_quantize(W, nbits, group, iters=0)
    rng = np.random.default_rng(41)
    sample = np.sort(rng.choice(rows, 48, replace=False))
    Wn = W[torch.from_numpy(sample).cuda()].cpu().numpy()
    ref = oracle.quantize(Wn, nbits, group, iters=0)
    gs = cols // group
    sc = q.scale.view(-1).cpu().numpy().reshape(rows, gs)[sample].reshape(-1)
    zf = q.zero_f32.view(-1).cpu().numpy().reshape(rows, gs)[sample].reshape(-1)
    assert np.array_equal(sc.view(np.uint16), ref["scale"].view(np.uint16))
    assert np.max(np.abs(zf - ref["zero_f32"])) <= ZERO_TOL
    g_idx = (sample[:, None] * gs + np.arange(gs)[None, :]).reshape(-1)
    codes = group_codes(q.packed.cpu().numpy(), nbits, group, g_idx).reshape(-1)
    assert np.array_equal(codes, ref["codes"])
    assert np.all(q.iters.view(-1).cpu().numpy() == 0)
