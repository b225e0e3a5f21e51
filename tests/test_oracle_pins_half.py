"""Pins of the oracle's half-precision solver to facts outside itself (CPU).

"Half-Quadratic Quantization of Large Machine Learning Models", section 2.2
(the implementation holds 1/s, "more stable in half precision") and section 3
(the whole solve runs on the GPU in half precision).  The readings the oracle
takes -- every element-wise step rounded once to fp16, reductions accumulated
in binary32 and rounded once to fp16, the error compared as the fp16 group
mean, binary32 hyper-parameters, and the fp16 range bounds outside which a
group is solved in single precision -- are stated in its source.  The checks
below use numpy's float16 arithmetic (each operation correctly rounded), fp64
recomputations with derived rounding bounds, brute-force search and special
cases; none of them calls the half-precision solver's own helpers.
"""
import numpy as np
import pytest

import oracle
import synth

U16 = 2.0 ** -11          # unit roundoff of fp16


def _groups(seed, n, G, std=0.02):
    W = synth.student_t_host((n, G), seed=seed, stream=77, std=std)
    return W.astype(np.float16).astype(np.float32)


def _is_f16(x):
    x = np.asarray(x, np.float32)
    fin = np.isfinite(x)
    return np.array_equal(x[fin].astype(np.float16).astype(np.float32), x[fin])


# ------------------------------------------------------------------ P1 (fp16)
@pytest.mark.parametrize("G", [8, 16])
def test_half_sp2_update_is_argmin_within_fp16_rounding(G):
    """Section 2.2: each z update is argmin_z 1/2 ||s(Wq - z) - (W - W_e)||^2
    for the codes and W_e of the accepted step, found here by fp64 grid search.
    The fp16 update may differ from it only by fp16 roundings: 1/s (one), W - W_e
    and its product with 1/s (two more), the code difference, and the final
    rounding of the mean:
        |z16 - z*| <= 2^-11 (3.01 max|(W - W_e)/s| + 1.01 max|term| + 1.01 |z*|)."""
    W = _groups(11, 24, G, std=1.5)
    checked = 0
    for w in W:
        tr = oracle.trace_group(w, 4, iters=6, precision="fp16")
        assert tr["half"]
        s = float(tr["s"])
        for t in range(min(tr["accepted"], tr["evaluations"] - 1)):
            q, we, z16 = tr["q"][t].astype(np.float64), tr["we"][t].astype(np.float64), \
                float(tr["z"][t + 1])
            r = w.astype(np.float64) - we
            grid = np.arange(-60.0, 60.0, 1e-3)
            J = ((s * (q[None, :] - grid[:, None]) - r[None, :]) ** 2).sum(1)
            zc = grid[np.argmin(J)]
            fine = np.arange(zc - 2e-3, zc + 2e-3, 1e-6)
            J = ((s * (q[None, :] - fine[:, None]) - r[None, :]) ** 2).sum(1)
            zg = fine[np.argmin(J)]
            term = q - r / s
            bound = U16 * (3.01 * np.abs(r / s).max() + 1.01 * np.abs(term).max()
                           + 1.01 * abs(zg)) + 2e-6
            assert abs(z16 - zg) <= bound, (t, z16, zg, bound)
            checked += 1
    assert checked >= 24


# ------------------------------------------------------------------ P2 (fp16)
@pytest.mark.parametrize("beta", [0.5, 1.0, 3.0])
def test_half_shrink_p1_is_fp16_soft_threshold(beta):
    """Section 2.1: at p = 1 the generalised shrink is soft-thresholding; in half
    precision, sign(d) max(fp16(|d| - fp16(1/beta_t)), 0) with numpy's fp16
    subtraction.  Checked on every accepted step of unit-scale groups, where
    the threshold is active."""
    W = _groups(12, 40, 64, std=2.0)
    seen_active = 0
    for w in W:
        tr = oracle.trace_group(w, 3, p=1.0, beta=beta, iters=5, precision="fp16")
        assert tr["half"]
        for t in range(tr["accepted"]):
            d = tr["d"][t].astype(np.float16)
            thr = np.float16(np.float32(1.0) / np.float32(tr["beta"][t]))
            y = (np.abs(d) - thr).astype(np.float16)
            ref = np.where(y > 0, y, np.float16(0)).astype(np.float32) * np.sign(d).astype(
                np.float32)
            got = tr["we"][t]
            assert np.array_equal(np.abs(got), np.abs(ref)), t
            assert np.all((got == 0) | (np.sign(got) == np.sign(d))), t
            seen_active += int((got != 0).sum())
    assert seen_active > 100


# ------------------------------------------------------------------ P3 (fp16)
@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (8, 128), (1, 32)])
def test_half_residual_within_half_step(nbits, G):
    """Section 2: W - Q^-1(Q(W)) stays within half a step for weights whose
    W/s + z lies in [-1/2, L + 1/2], up to fp16 roundings of 1/s, W/s, the sum
    with z, the code difference, its product with s and the final difference:
        |d| <= (s/2 + 2^-10 |W| + 2^-11 s |v| + 2^-10 s |Wq - z|)(1 + 2^-10)."""
    L = (1 << nbits) - 1
    W = _groups(13, 30, G)
    n = 0
    for w in W:
        tr = oracle.trace_group(w, nbits, iters=20, precision="fp16")
        assert tr["half"]
        s = float(tr["s"])
        w64 = w.astype(np.float64)
        for t in range(tr["evaluations"]):
            z = float(tr["z"][t])
            v = w64 / s + z
            inside = (v >= -0.5 + 1e-3) & (v <= L + 0.5 - 1e-3)
            q = tr["q"][t].astype(np.float64)
            bound = (s / 2 + 2 * U16 * np.abs(w64) + U16 * s * np.abs(v)
                     + 2 * U16 * s * np.abs(q - z)) * (1 + 2 * U16)
            d = np.abs(tr["d"][t].astype(np.float64))
            assert np.all(d[inside] <= bound[inside]), t
            n += int(inside.sum())
    assert n > 1000


# ------------------------------------------------------------------ P4 (fp16)
@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (2, 128), (4, 16), (8, 128),
                                     (1, 64)])
def test_half_error_sequence_and_early_stop(nbits, G):
    """Section 4.1: the solver stops as soon as the error stops improving.  The
    recorded fp16 errors must fall strictly over the accepted steps, the first
    non-decrease must stop the group, the best z must be the last accepted
    one, and each recorded error must be the mean |d|^p of its residual up to
    the fp16 roundings of each power and of the mean (plus the table power's
    few binary32 ulps):  |e - mean|d|^p| <= 2^-11 (2.01 mean|d|^p) + 2^-24.
    The residual itself must be W - s(Wq - z) up to its three fp16 roundings."""
    W = _groups(14, 40, G)
    for w in W:
        tr = oracle.trace_group(w, nbits, iters=20, precision="fp16")
        assert tr["half"]
        e, ne, na = tr["e"], tr["evaluations"], tr["accepted"]
        assert np.all(np.diff(e[:na]) < 0)
        if ne > na:
            assert not (e[na] < e[na - 1] if na else False) and ne == na + 1
        else:
            assert ne == 20
        if na:
            assert tr["z_best"] == tr["z"][na - 1] and tr["e_best"] == e[na - 1]
        s = float(tr["s"])
        w64 = w.astype(np.float64)
        for t in range(ne):
            d = tr["d"][t].astype(np.float64)
            m = float(np.mean(np.abs(d) ** 0.7))
            assert abs(float(e[t]) - m) <= U16 * 2.01 * m + 2.0 ** -24, (t, e[t], m)
            qz = tr["q"][t].astype(np.float64) - float(tr["z"][t])
            exact = w64 - s * qz
            assert np.all(np.abs(d - exact) <= 2 * U16 * s * np.abs(qz) * 1.001
                          + U16 * np.abs(d) + 2.0 ** -25), t


def test_half_values_are_fp16_numbers():
    """Section 3: the solve runs in half precision, so every value the solver
    forms -- s, 1/s, each z and error, each code, residual and W_e -- must be an
    fp16 number (a missing rounding step would show here)."""
    W = _groups(15, 20, 64, std=1.0)
    for w in W:
        tr = oracle.trace_group(w, 4, iters=10, precision="fp16")
        assert tr["half"]
        ne, na = tr["evaluations"], tr["accepted"]
        for x in (tr["s"], tr["inv"], tr["z0"], tr["z_best"], tr["e_best"], tr["z"][:ne],
                  tr["e"][:ne], tr["q"][:ne], tr["d"][:ne], tr["we"][:na]):
            assert _is_f16(x)


# ------------------------------------------------------------------ P5 (fp16)
@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (8, 128), (1, 16)])
def test_half_zero_iterations_is_fp16_minmax_rtn(nbits, G):
    """iters = 0 is min-max round-to-nearest in half precision, written here in
    numpy float16 arithmetic: s = (max - min)/L, 1/s, z = -min (1/s),
    codes = clip(rint(W (1/s) + z), 0, L) -- each operation rounded to fp16."""
    L = np.float16((1 << nbits) - 1)
    W = synth.student_t_host((64, 4 * G), seed=16, stream=nbits).astype(np.float16)
    r = oracle.quantize(W, nbits, G, iters=0, precision="fp16")
    g = W.reshape(-1, G)
    mn, mx = g.min(1), g.max(1)
    s = ((mx - mn) / L).astype(np.float16)
    inv = (np.float16(1) / s).astype(np.float16)
    z = -(mn * inv).astype(np.float16)
    v = ((g * inv[:, None]).astype(np.float16) + z[:, None]).astype(np.float16)
    codes = np.clip(np.rint(v.astype(np.float32)), 0, float(L)).astype(np.uint8)
    assert r["half"].all()
    assert np.array_equal(r["scale"].view(np.uint16), s.view(np.uint16))
    assert np.array_equal(r["zero"].view(np.uint16), z.view(np.uint16))
    assert np.array_equal(r["codes"], codes.reshape(-1))
    assert np.all(np.isinf(r["err"])) and np.all(r["iters"] == 0)


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
def test_half_constant_groups_reconstruct_exactly(nbits):
    """A constant group (s = 1/s = 1, z = -min) reconstructs exactly in fp16."""
    vals = np.array([0.0, -0.0, 1.0, -3.5, 0.0123, 6.0e-8, 8000.0, -60000.0], np.float16)
    W = np.repeat(vals, 64).astype(np.float16)
    r = oracle.quantize(W, nbits, 64, precision="fp16")
    Wh = oracle.dequantize(r["codes"], r["scale"], r["zero"], 64)
    assert r["half"].all()
    assert np.array_equal(Wh.astype(np.float32), W.astype(np.float32))


def test_half_fixed_point_stops():
    """If the codes and z repeat, the error repeats and the group stops (section
    4.1's early exit): a group already at a fixed point stops after one
    accepted step with the z it started from."""
    w = (np.arange(64, dtype=np.float32) % 16) * np.float32(0.0625) - np.float32(0.5)
    w = w.astype(np.float16).astype(np.float32)
    tr = oracle.trace_group(w, 4, iters=20, precision="fp16")
    assert tr["half"] and tr["accepted"] == 1 and tr["evaluations"] == 2
    assert tr["z"][1] == tr["z"][0] and tr["e"][1] == tr["e"][0] == 0


# ------------------------------------------------------------ fp16 bounds
@pytest.mark.parametrize("nbits,vals,half", [
    (4, [8192.0, 8100.0], True),       # largest |W| at the bound
    (4, [8200.0, 8100.0], False),      # beyond it
    (4, [1.0, 1.0 + 2 ** -10], True),  # max|W| (1/s) = 15 * 1024 = 15360 <= 2^14
    (8, [1.0, 1.0 + 2 ** -10], False),  # 255 * 1024 > 2^14
    (3, [0.0, 2.0 ** -24], False),     # s rounds to zero
    (2, [-1.0, 1.0], True)])
def test_half_bounds_fall_back_to_single_precision(nbits, vals, half):
    """Groups whose fp16 intermediates could overflow (largest |W| above 8192, s
    rounding to zero, or max|W| (1/s) above 2^14) are solved by the
    single-precision solver, whose results they must then equal exactly."""
    G = 16
    w = np.array([vals[i % 2] for i in range(G)], np.float16)
    r16 = oracle.quantize(w, nbits, G, precision="fp16")
    assert bool(r16["half"][0]) is half
    if not half:
        r32 = oracle.quantize(w, nbits, G)
        for k in ("codes", "scale", "zero", "zero_f32", "err", "iters"):
            assert np.array_equal(np.asarray(r16[k]).view(np.uint8),
                                  np.asarray(r32[k]).view(np.uint8)), k


@pytest.mark.parametrize("nbits,G", [(4, 64), (3, 64), (2, 32), (2, 128), (1, 64)])
def test_half_solver_close_to_single_precision(nbits, G):
    """The half-precision solve reaches nearly the same l_p error as the
    single-precision one on the synthetic weights (both ahead of RTN)."""
    W = synth.student_t_host((128, 1024), seed=17, stream=G).astype(np.float16)
    r16 = oracle.quantize(W, nbits, G, precision="fp16")
    r32 = oracle.quantize(W, nbits, G)
    rtn = oracle.quantize(W, nbits, G, iters=0)
    e = {k: oracle.lp_error(W, oracle.dequantize(r["codes"], r["scale"], r["zero"], G))
         for k, r in (("16", r16), ("32", r32), ("rtn", rtn))}
    assert r16["half"].all()
    assert e["16"] <= 1.01 * e["32"] and e["16"] < e["rtn"], e


def _pairwise32(x):
    x = np.asarray(x, np.float32)
    while x.size > 1:
        x = (x[: x.size // 2] + x[x.size // 2:]).astype(np.float32) if x.size > 2 else \
            np.array([np.float32(x[0]) + np.float32(x[1])], np.float32)
    return np.float32(x[0])


@pytest.mark.parametrize("nbits,G", [(4, 64), (3, 64), (2, 32), (8, 128), (1, 16)])
@pytest.mark.parametrize("std", [0.02, 1.5])
def test_half_each_evaluation_is_q_and_q_inverse_in_fp16(nbits, G, std):
    """Section 2's operators in half precision, with numpy's float16 arithmetic
    (each operation correctly rounded): the codes of evaluation t are
    Q_z(W) = clip(rint(fp16(fp16(W (1/s)) + z_t)), 0, L), its residual is
    fp16(W - fp16(s fp16(Wq - z_t))), its error is the fp16 mean of the
    fp16-rounded powers |d|^p (binary32 pairwise sum; the power itself from the
    separately pinned table-driven powp), and the final codes are those of the
    best evaluation."""
    L = (1 << nbits) - 1
    W = _groups(18, 16, G, std=std)
    for w in W:
        tr = oracle.trace_group(w, nbits, iters=20, precision="fp16")
        assert tr["half"]
        w16 = w.astype(np.float16)
        s16, inv16 = np.float16(tr["s"]), np.float16(tr["inv"])
        u = (w16 * inv16).astype(np.float16)
        for t in range(tr["evaluations"]):
            z16 = np.float16(tr["z"][t])
            v = (u + z16).astype(np.float16)
            q = np.clip(np.rint(v.astype(np.float32)), 0, L).astype(np.float32)
            assert np.array_equal(tr["q"][t], q), t
            d = (w16 - (s16 * (q.astype(np.float16) - z16).astype(np.float16)).astype(
                np.float16)).astype(np.float16)
            assert np.array_equal(tr["d"][t], d.astype(np.float32)), t
            pw = oracle.powp(np.abs(d.astype(np.float32)), 0.7).astype(np.float16)
            e = np.float16(_pairwise32(pw.astype(np.float32)) * np.float32(1.0 / G))
            assert tr["e"][t] == np.float32(e), t
        na = tr["accepted"]
        if na:
            assert np.array_equal(tr["codes"].astype(np.float32), tr["q"][na - 1])
