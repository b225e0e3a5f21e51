"""Pins of the CPU oracle to facts outside itself (run on CPU, no GPU).

Each test names the passage of "Half-Quadratic Quantization of Large Machine
Learning Models" (sections 2, 2.1, 2.2, 4.1) or the mathematical fact it uses.
"""
import decimal
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _groups(seed, n, G, std=0.02):
    W = synth.student_t_host((n, G), seed=seed, stream=99, std=std)
    return W.astype(np.float32)


# --------------------------------------------------------------------------- P1
@pytest.mark.parametrize("G", [8, 16])
def test_sp2_update_is_argmin_by_grid_search(G):
    """Section 2.2: z(t+1) = argmin_z 1/2 || s(Wq - z) - (W - W_e) ||^2, found here
    by brute-force fp64 grid search instead of the closed-form mean."""
    rng = np.random.default_rng(1)
    for trial in range(6):
        s = np.float32(rng.uniform(0.002, 0.05))
        inv = np.float32(1) / s
        w = (rng.standard_normal(G) * 0.02).astype(np.float32)
        q = rng.integers(0, 16, G).astype(np.float32)
        we = np.where(rng.random(G) < 0.3, rng.standard_normal(G) * 0.01, 0).astype(np.float32)
        z = float(oracle.z_update(w, q, we, inv))
        sd, wd, qd, wed = float(s), w.astype(np.float64), q.astype(np.float64), we.astype(np.float64)
        # coarse then fine grid, 1e-6 resolution around the coarse optimum
        grid = np.arange(-40.0, 40.0, 1e-3)
        J = ((sd * (qd[None, :] - grid[:, None]) - (wd - wed)[None, :]) ** 2).sum(1)
        zc = grid[np.argmin(J)]
        fine = np.arange(zc - 2e-3, zc + 2e-3, 1e-6)
        J = ((sd * (qd[None, :] - fine[:, None]) - (wd - wed)[None, :]) ** 2).sum(1)
        zg = fine[np.argmin(J)]
        assert abs(z - zg) <= 2e-6 + 2e-6 * abs(zg), (trial, z, zg)


# --------------------------------------------------------------------------- P2
@pytest.mark.parametrize("beta", [0.5, 1.0, 1.01 ** 7, 3.0])
def test_shrink_p1_is_soft_threshold(beta):
    """Section 2.1: for the l1 norm the proximal solution is soft-thresholding,
    sign(x) max(|x| - 1/beta, 0); the oracle's generalised shrink at p = 1 must
    equal it bit for bit (|x|^0 == 1 exactly)."""
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 3,
                        np.array([0.0, -0.0, 1 / beta, -1 / beta], np.float32)])
    we = oracle.shrink(x, 1.0, beta)
    thr = np.float32(1) / np.float32(beta)
    ref = np.sign(x) * np.maximum(np.abs(x) - thr, np.float32(0))
    assert np.array_equal(we, ref.astype(np.float32))


@pytest.mark.parametrize("p", [0.7, 0.5, 0.9])
@pytest.mark.parametrize("beta", [1.0, 1.5, 10.0])
def test_shrink_threshold_closed_form(p, beta):
    """Section 2.1: shrink_lp(x) is non-zero exactly when |x| - |x|^(p-1)/beta > 0,
    i.e. when |x| > T = beta^(-1/(2-p)); it keeps the sign of x and shrinks |x|."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(50000) * 2).astype(np.float32)
    T = beta ** (-1.0 / (2.0 - p))
    keep = np.abs(np.abs(x.astype(np.float64)) / T - 1) > 1e-4
    x = x[keep]
    we = oracle.shrink(x, p, beta)
    ax = np.abs(x.astype(np.float64))
    active = ax > T
    assert np.all((we != 0) == active)
    assert np.all(np.sign(we[active]) == np.sign(x[active]))
    assert np.all(np.abs(we) <= np.abs(x))
    ref = np.sign(x[active]) * (ax[active] - ax[active] ** (p - 1) / beta)
    np.testing.assert_allclose(we[active], ref, rtol=3e-6, atol=2e-7)


# --------------------------------------------------------------------------- P3
@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (2, 128)])
def test_residual_within_half_step(nbits, G):
    """Section 2: Wq = round(W/s + z), W_hat = s(Wq - z).  With W_e = 0, every
    weight whose W/s + z lies in [-1/2, L + 1/2] is reconstructed within s/2."""
    L = 2 ** nbits - 1
    W = _groups(4, 40, G)
    for w in W:
        tr = oracle.trace_group(w, nbits)
        s = float(tr["s"])
        for t in range(tr["evaluations"]):
            u = w.astype(np.float64) / s + float(tr["z"][t])
            inr = (u >= -0.5 + 1e-5) & (u <= L + 0.5 - 1e-5)
            assert np.all(np.abs(tr["d"][t][inr]) <= s / 2 * (1 + 1e-5))
            # the code is the nearest level, clamped
            assert np.array_equal(tr["q"][t], np.clip(np.rint(u), 0, L)) or \
                np.all(np.abs(np.abs(u - np.floor(u)) - 0.5)[tr["q"][t] != np.clip(np.rint(u), 0, L)] < 1e-5)


# --------------------------------------------------------------------------- P4
@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (2, 128), (4, 16)])
def test_error_sequence_and_early_stop(nbits, G):
    """Section 4.1: the solver runs at most 20 iterations and exits once the error
    stops improving.  Accepted errors fall strictly; the first non-decrease ends
    the group; z_best is the z of the last accepted evaluation; each recorded
    error equals sum |W - s(round(W/s+z) - z)|^p recomputed in fp64."""
    W = _groups(5, 60, G)
    p = 0.7
    for w in W:
        tr = oracle.trace_group(w, nbits, p=p)
        e, z, n, a = tr["e"], tr["z"], tr["evaluations"], tr["accepted"]
        assert a <= 20 and n == a + (1 if a < 20 else 0)
        assert np.all(np.diff(e[:a]) < 0)
        if a < 20:
            assert not (e[a] < e[a - 1] if a > 0 else False)
        if a > 0:
            assert tr["z_best"] == z[a - 1] and tr["e_best"] == e[a - 1]
        assert e[0] >= tr["e_best"]          # never worse than min-max RTN
        assert z[0] == tr["z0"]
        s = float(tr["s"])
        L = 2 ** nbits - 1
        wd = w.astype(np.float64)
        for t in range(n):
            q = np.clip(np.rint(wd / s + float(z[t])), 0, L)
            ref = np.sum(np.abs(wd - s * (q - float(z[t]))) ** p)
            assert abs(float(e[t]) - ref) <= 2e-5 * ref + 1e-30


def test_beta_schedule():
    """Section 2: beta(t+1) = kappa * beta(t), starting from beta = 1, kappa = 1.01."""
    rng = np.random.default_rng(6)
    w = (rng.standard_normal(64) * 2).astype(np.float32)  # unit scale: many iterations
    tr = oracle.trace_group(w, 2, beta=1.0, kappa=1.01)
    for t, b in enumerate(tr["beta"]):
        assert abs(float(b) - 1.01 ** t) <= 1e-6 * 1.01 ** t * (t + 1)


def test_components_compose_into_the_solver():
    """The recorded iterations are exactly sp1 then sp2 of the component
    functions pinned above (shrink of the residual with beta(t), then the mean)."""
    rng = np.random.default_rng(7)
    for k in range(30):
        w = (rng.standard_normal(64) * (2.0 if k % 2 else 0.02)).astype(np.float32)
        tr = oracle.trace_group(w, 3)
        for t in range(tr["accepted"]):
            we = oracle.shrink(tr["d"][t], 0.7, float(tr["beta"][t]))
            assert np.array_equal(we, tr["we"][t])
            z1 = oracle.z_update(w, tr["q"][t], we, float(tr["inv"]))
            if t + 1 < tr["evaluations"]:
                assert z1 == tr["z"][t + 1]


# --------------------------------------------------------------------------- P5
@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (2, 128), (4, 16)])
def test_zero_iterations_is_minmax_rtn(nbits, G):
    """iters = 0 is textbook asymmetric min-max round-to-nearest: scale =
    (max - min)/(2^b - 1), zero = -min/scale, code = clip(round(W/scale + zero))."""
    W = synth.student_t_host((256, G), seed=8, stream=3).astype(np.float16)
    r = oracle.quantize(W, nbits, G, iters=0)
    L = 2 ** nbits - 1
    w = W.astype(np.float64)
    mn, mx = w.min(1, keepdims=True), w.max(1, keepdims=True)
    scale = (mx - mn) / L
    zero = -mn / scale
    u = w / scale + zero
    codes = np.clip(np.rint(u), 0, L).reshape(-1)
    tie = (np.abs(np.abs(u - np.floor(u)) - 0.5) < 1e-5).reshape(-1)
    assert np.all((r["codes"] == codes) | tie)
    assert np.mean(tie) < 1e-3          # differences only at exact half-way ties
    np.testing.assert_allclose(r["scale_f32"], scale.ravel(), rtol=1e-7)
    np.testing.assert_allclose(r["zero_f32"], zero.ravel(), rtol=1e-6, atol=1e-6)
    assert np.all(r["iters"] == 0)


# --------------------------------------------------------------------------- P6
@pytest.mark.parametrize("nbits", [2, 3, 4])
def test_constant_groups_reconstruct_exactly(nbits):
    """A group with max == min has a single level; Q^-1(Q(W)) must equal W."""
    G = 32
    vals = np.array([0.0, 1.0, -0.015625, 3.5, -65504.0, 6e-8, 0.0999755859375], np.float16)
    W = np.repeat(vals, G).astype(np.float16)
    r = oracle.quantize(W, nbits, G)
    Wh = oracle.dequantize(r["codes"], r["scale"], r["zero"], G)
    assert np.array_equal(Wh.view(np.uint16) & 0x7FFF, W.view(np.uint16) & 0x7FFF)
    assert np.array_equal(Wh.astype(np.float32), W.astype(np.float32))
    assert np.all(r["scale_f32"] == 1.0)


# --------------------------------------------------------------------------- P7
def _golden_pack():
    out = []
    with open(os.path.join(GOLDEN, "pack_layout.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            nb, codes, hexb = (x.strip() for x in line.split("|"))
            out.append((int(nb), [int(c) for c in codes.split()], bytes.fromhex(hexb)))
    return out


@pytest.mark.parametrize("case", _golden_pack())
def test_pack_golden(case):
    nbits, codes, packed = case
    got = oracle.pack(np.array(codes, np.uint8), nbits)
    assert got.tobytes() == packed
    assert oracle.unpack(got, len(codes), nbits).tolist() == codes


@pytest.mark.parametrize("nbits", [2, 3, 4])
def test_pack_roundtrip_all_values_and_positions(nbits):
    rng = np.random.default_rng(9)
    for n in [1, 7, 10, 31, 320, 1001]:
        codes = rng.integers(0, 2 ** nbits, n).astype(np.uint8)
        pk = oracle.pack(codes, nbits)
        assert pk.size == oracle.packed_bytes(n, nbits)
        assert np.array_equal(oracle.unpack(pk, n, nbits), codes)
    # every value at every slot of a word
    per = {4: 8, 2: 16, 3: 10}[nbits]
    for v in range(2 ** nbits):
        for pos in range(per):
            codes = np.zeros(per, np.uint8)
            codes[pos] = v
            word = int.from_bytes(oracle.pack(codes, nbits)[:4].tobytes(), "little")
            assert word == v << (nbits * pos)


# --------------------------------------------------------------------------- P8
def test_fixed_point_stops():
    """Section 2.2: with Wq unchanged between two evaluations and W_e = 0 the mean
    gives the same z, so the error repeats and the group stops on equality."""
    W = _groups(10, 300, 64)
    seen = 0
    for w in W:
        tr = oracle.trace_group(w, 4)
        q, a, n = tr["q"], tr["accepted"], tr["evaluations"]
        for t in range(a - 1):
            if np.array_equal(q[t], q[t + 1]) and np.all(tr["we"][t] == 0) and t + 2 < n + 1:
                assert t + 2 == n - 1 or t + 2 >= n
                if t + 2 < n:
                    assert tr["z"][t + 2] == tr["z"][t + 1]
                    assert tr["e"][t + 2] == tr["e"][t + 1]
                seen += 1
    assert seen > 10


# --------------------------------------------------------------------------- P9
def _ulp32(x):
    x = np.abs(np.asarray(x, np.float32))
    return np.spacing(x).astype(np.float64)


@pytest.mark.parametrize("p", [0.7, -0.3, 0.5, 0.1, -0.9, 1.0, 0.999])
def test_powp_accuracy(p):
    """|x|^p of the l_p error (section 2) and of the shrink (section 2.1): the
    table-driven power must stay within 4 ulp of the fp64 library pow."""
    rng = np.random.default_rng(11)
    x = np.concatenate([
        np.exp2(rng.uniform(-126, 127, 400000)).astype(np.float32),
        rng.uniform(0, 1, 200000).astype(np.float32),
        rng.uniform(1e-4, 0.2, 200000).astype(np.float32),
        np.float32(1) + np.arange(-512, 512, dtype=np.float32) * np.float32(2 ** -23),
    ])
    x = x[(x >= np.float32(2 ** -126)) & np.isfinite(x)]
    y = oracle.powp(x, p).astype(np.float64)
    ref = np.power(x.astype(np.float64), float(np.float32(p)))
    fin = np.isfinite(ref) & (ref < 3e38) & (ref > 1.2e-38)
    err = np.abs(y[fin] - ref[fin]) / _ulp32(ref[fin].astype(np.float32))
    assert err.max() <= 4.0, err.max()


def test_powp_special_values():
    tiny = np.array([0.0, 1e-45, 1e-40, 2 ** -127], np.float32)
    assert np.all(oracle.powp(tiny, 0.7) == 0)
    assert np.all(np.isinf(oracle.powp(tiny, -0.3)))
    x = np.array([0.0, 1e-40, 1e-3, 1.0, 7.5, 65504.0], np.float32)
    assert np.all(oracle.powp(x, 0.0) == 1.0)
    assert oracle.powp(np.array([1.0], np.float32), 0.7)[0] == pytest.approx(1.0, rel=2e-7)


def _exact_pow2(y: decimal.Decimal) -> decimal.Decimal:
    return (y * decimal.Decimal(2).ln()).exp()


@pytest.mark.parametrize("p", [0.7, -0.3])
def test_powp_table_entries_correctly_rounded(p):
    """The 2^(p k) and c_j^p entries are the binary32 values nearest to the exact
    powers (50-digit decimal arithmetic, independent of the C library)."""
    decimal.getcontext().prec = 50
    tab = oracle.powp_table(p)
    pd = decimal.Decimal(float(np.float32(p)))
    bad = 0
    for e in range(1, 255):
        exact = _exact_pow2(pd * (e - 127))
        got = decimal.Decimal(float(tab["two_pk"][e]))
        ulp = decimal.Decimal(float(np.spacing(np.float32(float(exact)))))
        bad += abs(got - exact) > ulp / 2
    for j in range(32):
        c = 1 + decimal.Decimal(2 * j + 1) / 64
        exact = (pd * c.ln()).exp()
        got = decimal.Decimal(float(tab["cj_p"][j]))
        ulp = decimal.Decimal(float(np.spacing(np.float32(float(exact)))))
        bad += abs(got - exact) > ulp / 2
        assert tab["inv_cj"][j] == np.float32(1) / np.float32(float(c))
    assert bad == 0


def test_psum_is_pairwise_over_contiguous_halves():
    """PSUM(x[0..n)) = PSUM(first half) + PSUM(second half): a sum whose value
    depends on the order tells the order apart."""
    x = np.array([1.0, 2.0 ** 24, 1.0, -(2.0 ** 24)], np.float32)
    assert oracle.psum(x) == np.float32(1.0)        # sequential: 0, strided: 2
    rng = np.random.default_rng(12)
    for n in [2, 8, 64, 256]:
        v = (rng.standard_normal(n) * 10 ** rng.uniform(-3, 3, n)).astype(np.float32)

        def pw(a):
            return a[0] if a.size == 1 else np.float32(pw(a[: a.size // 2]) + pw(a[a.size // 2:]))
        assert oracle.psum(v) == pw(v)


def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(13)
    x = np.concatenate([(rng.standard_normal(100000) * 10 ** rng.uniform(-9, 5, 100000)),
                        [65504.0, 65519.99, 65520.0, 6e-8, 2.98e-8, 1.0 + 2 ** -11,
                         1.0 + 3 * 2 ** -11, -0.0]]).astype(np.float32)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16)
    assert np.array_equal(oracle.f32_to_f16(x).view(np.uint16), ref.view(np.uint16))


# ----------------------------------------------------------------- whole pipeline
def test_matrix_equals_independent_groups():
    """Early stopping is per group: quantizing a matrix equals solving each of its
    groups alone."""
    W = synth.student_t_host((16, 128), seed=14, stream=1)
    r = oracle.quantize(W, 3, 64, threads=3)
    flat = W.astype(np.float32).reshape(-1, 64)
    for g, w in enumerate(flat):
        tr = oracle.trace_group(w, 3)
        assert np.array_equal(tr["codes"], r["codes"][g * 64:(g + 1) * 64])
        assert tr["z_best"] == r["zero_f32"][g]
        assert tr["accepted"] == r["iters"][g]
        assert np.float16(tr["s"]) == r["scale"][g]


@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64)])
def test_hqq_not_worse_than_rtn(nbits, G):
    """Per group, the chosen z never has a larger l_p error than the min-max z it
    starts from (fp64 recomputation from the final codes, fp32 scale and zero)."""
    W = synth.student_t_host((128, 256), seed=15, stream=2)
    r = oracle.quantize(W, nbits, G)
    r0 = oracle.quantize(W, nbits, G, iters=0)
    w = W.astype(np.float64).reshape(-1, G)

    def err(res):
        c = res["codes"].reshape(-1, G).astype(np.float64)
        s = res["scale_f32"].astype(np.float64)[:, None]
        z = res["zero_f32"].astype(np.float64)[:, None]
        return (np.abs(w - s * (c - z)) ** 0.7).sum(1)
    e, e0 = err(r), err(r0)
    assert np.all(e <= e0 * (1 + 1e-5))
    assert e.sum() < e0.sum() * 0.995


def test_dequantize_definition():
    """Q^-1(Wq) = s(Wq - z) with the stored fp16 s and z, rounded to fp16."""
    rng = np.random.default_rng(16)
    G = 32
    codes = rng.integers(0, 16, 64 * G).astype(np.uint8)
    scale = (rng.uniform(1e-3, 0.1, 64)).astype(np.float16)
    zero = (rng.uniform(-2, 18, 64)).astype(np.float16)
    got = oracle.dequantize(codes, scale, zero, G)
    ref = ((codes.astype(np.float32) - np.repeat(zero.astype(np.float32), G))
           * np.repeat(scale.astype(np.float32), G)).astype(np.float16)
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))
