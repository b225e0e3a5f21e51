"""GPU parity of the half-precision solver (hqq_quantize_half, through the C
ABI) against the oracle's half-precision solver, element by element on the
same seeded inputs.

"Half-Quadratic Quantization of Large Machine Learning Models", section 2.2
(1/s held because it is more stable in half precision) and section 3 (the
whole solve in half precision).  Both sides follow the same readings of the
fp16 steps, so the tolerances are those of the single-precision path
(tests/_parity.py): scales bit-identical, z within 1e-4 code units (equal
expected), codes >= 99.99 % (100 % expected), per-tensor l_p error within
1e-4 relative; the recorded errors (fp16 group means) and accepted-iteration
counts identical, and the same groups solved in half precision.
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


def _check(W_dev, W_np, nbits, group, label, **kw):
    q = gpu_quantize(W_dev, nbits, group, precision="fp16", **kw)
    gq = to_np(q)
    ref = oracle.quantize(W_np, nbits, group, precision="fp16", **kw)
    st = compare_full(W_np, gq, ref, nbits, group, p=kw.get("p", 0.7), label=label)
    half = q.half.cpu().numpy().reshape(-1).astype(bool)
    assert np.array_equal(half, ref["half"]), f"{label}: half-precision groups differ"
    st["half_frac"] = float(half.mean()) if half.size else 1.0
    return gq, ref, st


# ---------------------------------------------------------------- the configs
def test_c1_1024_4bit_g64(hqq):
    W, Wn = _dev_weights((1024, 1024), seed=0)
    _, _, st = _check(W, Wn, 4, 64, "fp16 1024^2 4b g64")
    assert st["code_match"] == 1.0 and st["max_dz"] == 0.0 and st["half_frac"] == 1.0


@pytest.mark.parametrize("nbits,group", [(4, 64), (2, 32)])
def test_c2_4096(hqq, nbits, group):
    W, Wn = _dev_weights((4096, 4096), seed=1)
    _, _, st = _check(W, Wn, nbits, group, f"fp16 4096^2 {nbits}b g{group}")
    assert st["code_match"] == 1.0 and st["half_frac"] == 1.0


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("group", [16, 32, 64, 128, 256])
def test_all_formats_ragged(hqq, nbits, group):
    W, Wn = _dev_weights((37, 13 * group), seed=21, stream=nbits * 1000 + group)
    _, _, st = _check(W, Wn, nbits, group, f"fp16 ragged {nbits}b g{group}")
    assert st["code_match"] == 1.0


@pytest.mark.parametrize("shape", [(1, 64), (3, 64), (1, 640), (5, 192)])
@pytest.mark.parametrize("nbits", [1, 3, 4, 8])
def test_odd_shapes(hqq, shape, nbits):
    W, Wn = _dev_weights(shape, seed=22, stream=shape[0] * 7 + shape[1])
    _check(W, Wn, nbits, 64, f"fp16 shape {shape} {nbits}b")


# ------------------------------------------- adversarial groups and fp16 bounds
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
    r = np.full(G, 65504.0); r[::2] = -65504.0; rows.append(r)   # +-max fp16: single precision
    rows.append(np.where(np.arange(G) < G // 2, 1e-3, -1e-3))    # two levels
    r = rng.standard_normal(G); rows.append(r)                   # unit scale (shrink on)
    r = rng.standard_normal(G) * 10; rows.append(r)              # large scale
    rows.append(np.full(G, 6e-8))                                # constant subnormal
    r = np.zeros(G); r[1::2] = -0.0; r[::3] = 0.25; rows.append(r)  # signed zeros
    r = 1.0 + np.arange(G) % 2 * 2.0 ** -10; rows.append(r)      # range of one ulp near 1
    r = rng.standard_normal(G) * 3000 + 5000; rows.append(r)     # near the 8192 bound
    r = rng.standard_normal(G) * 100; r[0] = 9000.0; rows.append(r)  # beyond it
    return np.array(rows, np.float64).astype(np.float16)


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("group", [16, 64, 128])
def test_adversarial_groups_and_bounds(hqq, nbits, group):
    Wn = _adversarial(group)
    W = torch.from_numpy(Wn).cuda()
    _, ref, st = _check(W, Wn, nbits, group, f"fp16 adversarial {nbits}b g{group}")
    assert 0.0 < st["half_frac"] < 1.0         # both precisions occur in one launch


@pytest.mark.parametrize("nbits,group", [(4, 64), (2, 32), (3, 64), (8, 128), (1, 64)])
@pytest.mark.parametrize("std", [1.0, 3.0])
def test_shrink_active(hqq, nbits, group, std):
    """Unit-scale weights: the half-precision shrink is active (the exact fp16
    formula replaces the zero shortcut)."""
    W, Wn = _dev_weights((256, 1024), seed=24, stream=group, std=std)
    _, _, st = _check(W, Wn, nbits, group, f"fp16 std {std} {nbits}b g{group}")
    assert st["code_match"] == 1.0 and st["iters_equal"] == 1.0


@pytest.mark.parametrize("nbits,group", [(3, 64), (4, 64)])
@pytest.mark.parametrize("std", [0.02, 3.0])
def test_wide_ctas_full(hqq, nbits, group, std):
    """4096 x 8192: enough chunks for one 20-warp CTA per SM on a 148-SM B200;
    every group against the oracle's half-precision solver, shrink inactive
    and active."""
    W, Wn = _dev_weights((4096, 8192), seed=25, stream=nbits, std=std)
    _, _, st = _check(W, Wn, nbits, group, f"fp16 wide std {std} {nbits}b g{group}")
    assert st["code_match"] == 1.0 and st["iters_equal"] == 1.0


@pytest.mark.parametrize("kw", [
    dict(iters=0), dict(iters=1), dict(iters=255), dict(p=1.0), dict(p=0.5),
    dict(p=0.05), dict(beta=0.1), dict(beta=50.0), dict(kappa=1.5), dict(kappa=0.9),
    dict(p=1.0, beta=2.0, kappa=1.2, iters=40),
])
def test_solver_parameters(hqq, kw):
    W, Wn = _dev_weights((128, 1024), seed=25, stream=3, std=0.5)
    _, _, st = _check(W, Wn, 4, 64, f"fp16 params {kw}", **kw)
    assert st["code_match"] == 1.0


@pytest.mark.parametrize("nbits,group", [(4, 64), (4, 16), (3, 64), (2, 128), (8, 32), (1, 256)])
def test_multi_chunk_per_warp(hqq, nbits, group):
    """More chunks than resident warps: groups still running at the end of a
    chunk are carried to the next one (4 bits) or drained."""
    W, Wn = _dev_weights((2048, 8192), seed=30, stream=group * 10 + nbits)
    _, _, st = _check(W, Wn, nbits, group, f"fp16 multi-chunk {nbits}b g{group}")
    assert st["code_match"] == 1.0


def test_multi_chunk_mixed_precisions(hqq):
    """Groups beyond the fp16 bounds scattered through a matrix large enough
    for carried groups: each takes the single-precision solver inside the
    same warps as the half-precision ones."""
    W, Wn = _dev_weights((1024, 8192), seed=32, stream=1, std=1.0)
    rng = np.random.default_rng(5)
    Wn = Wn.copy()
    g = Wn.reshape(-1, 64)
    pick = rng.choice(g.shape[0], 3000, replace=False)
    g[pick, rng.integers(0, 64, pick.size)] = np.float16(9000.0)
    W = torch.from_numpy(Wn).cuda()
    _, _, st = _check(W, Wn, 4, 64, "fp16 mixed precisions")
    assert 0.95 < st["half_frac"] < 1.0 and st["code_match"] == 1.0


FULL = [
    ("70B gate 28672x8192 3b g64", (28672, 8192), 3, 64, 5, 4),
    ("8192x8192 2b g32", (8192, 8192), 2, 32, 3, 0),
    ("8192x8192 8b g128", (8192, 8192), 8, 128, 7, 0),
    ("7B up 11008x4096 4b g64", (11008, 4096), 4, 64, 2, 5),
]


@pytest.mark.parametrize("label,shape,nbits,group,seed,stream", FULL,
                         ids=[f[0] for f in FULL])
def test_full_size_sampled(hqq, label, shape, nbits, group, seed, stream):
    W = synth.student_t_device(shape, seed=seed, stream=stream)
    q = gpu_quantize(W, nbits, group, precision="fp16")
    torch.cuda.synchronize()
    n_groups = W.numel() // group
    rng = np.random.default_rng(seed * 100 + stream)
    g_idx = np.unique(np.concatenate([rng.integers(0, n_groups, 4000),
                                      [0, 1, n_groups - 1, n_groups - 2]]))
    sel = torch.from_numpy(g_idx).cuda()
    Wg = W.view(-1, group)[sel].cpu().numpy()
    ref = oracle.quantize(Wg, nbits, group, precision="fp16")
    codes = group_codes(q.packed.cpu().numpy(), nbits, group, g_idx)
    pick = lambda t: t.view(-1)[sel].cpu().numpy()
    assert np.array_equal(pick(q.err).view(np.uint32), ref["err"].view(np.uint32))
    assert np.array_equal(pick(q.scale).view(np.uint16), ref["scale"].view(np.uint16))
    assert np.max(np.abs(pick(q.zero_f32).astype(np.float64) - ref["zero_f32"])) <= ZERO_TOL
    assert np.mean(codes.reshape(-1) == ref["codes"]) >= CODE_MATCH
    assert np.array_equal(pick(q.iters), ref["iters"])
    assert np.array_equal(pick(q.half).astype(bool), ref["half"])


def test_half_bad_arguments_touch_nothing(hqq):
    import ctypes
    L = hqq._lib
    W = synth.student_t_device((64, 256), seed=27)
    packed = torch.full((64 * 256 // 2,), 0xAB, dtype=torch.uint8, device="cuda")
    scale = torch.full((64, 4), 7.0, dtype=torch.float16, device="cuda")
    zero = torch.full((64, 4), 7.0, dtype=torch.float16, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for over, want in [(dict(nbits=5), 3), (dict(group=48), 3), (dict(cols=250), 2),
                       (dict(p=0.0), 4), (dict(iters=256), 4), (dict(beta=float("nan")), 4)]:
        a = dict(rows=64, cols=256, nbits=4, group=64, p=0.7, beta=1.0, kappa=1.01, iters=20)
        a.update(over)
        st = L.hqq_quantize_half(P(W), a["rows"], a["cols"], a["nbits"], a["group"], a["p"],
                                 a["beta"], a["kappa"], a["iters"], P(packed), P(scale), P(zero),
                                 None, None, None, None, s)
        assert st == want, (over, st)
    torch.cuda.synchronize()
    assert torch.all(packed == 0xAB) and torch.all(scale == 7.0) and torch.all(zero == 7.0)
