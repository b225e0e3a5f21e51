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
@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (2, 128), (8, 128), (1, 32)])
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
@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (2, 128), (4, 16), (8, 128),
                                     (1, 64)])
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
@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (2, 128), (4, 16), (8, 128),
                                     (1, 64)])
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
@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
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


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
def test_pack_roundtrip_all_values_and_positions(nbits):
    rng = np.random.default_rng(9)
    for n in [1, 7, 10, 31, 320, 1001]:
        codes = rng.integers(0, 2 ** nbits, n).astype(np.uint8)
        pk = oracle.pack(codes, nbits)
        assert pk.size == oracle.packed_bytes(n, nbits)
        assert np.array_equal(oracle.unpack(pk, n, nbits), codes)
    # every value at every slot of a word
    per = {8: 4, 4: 8, 2: 16, 1: 32, 3: 10}[nbits]
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


@pytest.mark.parametrize("nbits,G", [(4, 64), (2, 32), (3, 64), (8, 128), (1, 64)])
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


# ------------------------------------------------------------ 8-bit meta data
def _meta_inputs(seed):
    """Realistic zero points and scales: those of HQQ-quantized synthetic weights."""
    W = synth.student_t_host((192, 1024), seed=seed, stream=11).astype(np.float16)
    r = oracle.quantize(W, 3, 64, iters=4)
    return r["zero"].copy(), r["scale"].copy()


@pytest.mark.parametrize("which", ["zero", "scale"])
@pytest.mark.parametrize("group", [0, 128, 100])
def test_meta_quantize_is_8bit_minmax_rtn(which, group):
    """Section 4.1 stores the zero points (no grouping) and, in the table's
    starred row, the scales (groups of 128) in 8 bits; with no optimisation this
    is textbook min-max round-to-nearest with 255 levels, checked here in fp64
    (ragged last group when 128 or 100 does not divide the length)."""
    zero, scale = _meta_inputs(21)
    x = (zero if which == "zero" else scale)[:700]
    r = oracle.meta_quantize(x, group)
    n = x.size
    ln = n if group == 0 else group
    xd = x.astype(np.float64)
    for gi, g0 in enumerate(range(0, n, ln)):
        seg = xd[g0:g0 + ln]
        mn, mx = seg.min(), seg.max()
        s = (mx - mn) / 255.0
        z = -mn / s
        u = seg / s + z
        codes = np.clip(np.rint(u), 0, 255)
        tie = np.abs(np.abs(u - np.floor(u)) - 0.5) < 1e-4
        got = r["codes"][g0:g0 + ln]
        assert np.all((got == codes) | tie), gi
        assert got.min() == 0 and got.max() == 255
        # stored fp16 values: the fp64 ones rounded to fp16 (one fp16 ulp slack
        # for the fp32 intermediate)
        for stored, exact in ((r["scale"][gi], s), (r["zero"][gi], z)):
            ref = np.float16(exact)
            ulp = np.spacing(np.abs(ref)).astype(np.float64)
            assert abs(float(stored) - exact) <= float(ulp), (gi, stored, exact)
    assert r["scale"].size == oracle.meta_groups(n, group)


def test_meta_group_semantics():
    """Group 0 is one group over the whole tensor; groups are independent runs
    of consecutive values, the last one shorter."""
    zero, _ = _meta_inputs(22)
    x = zero[:1000]
    a = oracle.meta_quantize(x, 0)
    b = oracle.meta_quantize(x, 1000)
    assert all(np.array_equal(a[k].view(np.uint8), b[k].view(np.uint8)) for k in a)
    c = oracle.meta_quantize(x, 128)
    for gi, g0 in enumerate(range(0, 1000, 128)):
        d = oracle.meta_quantize(x[g0:g0 + 128], 0)
        assert np.array_equal(c["codes"][g0:g0 + 128], d["codes"])
        assert c["scale"][gi] == d["scale"][0] and c["zero"][gi] == d["zero"][0]


def test_meta_constant_and_degenerate_groups():
    """A constant group has one level (s = 1) and restores exactly; an empty
    tensor has no groups."""
    vals = np.array([0.0, 3.5, -0.25, 7.0, 6e-8, 1000.0], np.float16)
    x = np.repeat(vals, 128)
    r = oracle.meta_quantize(x, 128)
    assert np.all(r["scale"] == 1.0) and np.all(r["codes"] == 0)
    y = oracle.meta_dequantize(r["codes"], r["scale"], r["zero"], 128)
    assert np.array_equal(y.astype(np.float32), x.astype(np.float32))
    e = oracle.meta_quantize(np.zeros(0, np.float16), 0)
    assert e["codes"].size == 0 and e["scale"].size == 0


def test_meta_dequantize_and_composition_definition():
    """Q^-1 on 8-bit codes is fp16((c - z) s) with the group's fp16 s and z
    (numpy fp32 here); weights with 8-bit zero points (and scales) are restored
    by restoring the zero points (and scales) first, then Q^-1 as usual."""
    zero, scale = _meta_inputs(23)
    zq = oracle.meta_quantize(zero, 0)
    sq = oracle.meta_quantize(scale, 128)
    n = zero.size
    zr = ((zq["codes"].astype(np.float32) - np.float32(zq["zero"][0]))
          * np.float32(zq["scale"][0])).astype(np.float16)
    got = oracle.meta_dequantize(zq["codes"], zq["scale"], zq["zero"], 0)
    assert np.array_equal(got.view(np.uint16), zr.view(np.uint16))
    gidx = np.arange(n) // 128
    sr = ((sq["codes"].astype(np.float32) - sq["zero"].astype(np.float32)[gidx])
          * sq["scale"].astype(np.float32)[gidx]).astype(np.float16)
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 8, n * 64).astype(np.uint8)
    w1 = oracle.dequantize_meta(codes, 64, zq, 0, scale=scale)
    assert np.array_equal(w1.view(np.uint16), oracle.dequantize(codes, scale, zr, 64).view(np.uint16))
    w2 = oracle.dequantize_meta(codes, 64, zq, 0, scale_q=sq, scale_group=128)
    assert np.array_equal(w2.view(np.uint16), oracle.dequantize(codes, sr, zr, 64).view(np.uint16))


def test_meta_zero_error_is_small_against_the_code_step():
    """8 bits for the zero points of a 3-bit matrix cost little: every restored
    zero point lies within half a step of the 8-bit grid of the stored fp16 s and
    z (plus the fp16 rounding of the result) of its original."""
    zero, _ = _meta_inputs(24)
    zq = oracle.meta_quantize(zero, 0)
    zr = oracle.meta_dequantize(zq["codes"], zq["scale"], zq["zero"], 0).astype(np.float64)
    s16 = float(zq["scale"][0])
    rng_ = float(zero.astype(np.float64).max() - zero.astype(np.float64).min())
    bound = s16 / 2 + 255 * abs(s16 - rng_ / 255) + abs(float(zq["zero"][0]) - float(
        -zero.astype(np.float64).min() / (rng_ / 255))) * s16 + np.spacing(np.float16(8.0))
    assert np.max(np.abs(zr - zero.astype(np.float64))) <= bound


# ------------------------------------------------- weight-only linear layer
def test_linear_is_x_times_w_transposed():
    """Y = X W_hat^T: with X the identity, row k of Y is column k of W_hat
    (output features along Y's columns), exactly; a plain triple loop on a tiny
    case gives the same fp64 values; the fp16 result is the fp64 one rounded
    once."""
    rng = np.random.default_rng(40)
    N, K = 24, 64
    W = synth.student_t_host((N, K), seed=40, stream=1).astype(np.float16)
    r = oracle.quantize(W, 4, 32, iters=3)
    Wh = oracle.dequantize(r["codes"], r["scale"], r["zero"], 32).reshape(N, K)
    eye = np.eye(K, dtype=np.float16)
    out = oracle.linear(eye, Wh)
    assert np.array_equal(out["y"], Wh.T)
    X = (rng.standard_normal((5, K))).astype(np.float16)
    out = oracle.linear(X, Wh)
    for m in range(5):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(X[m, k]) * float(Wh[n, k])
            assert abs(acc - out["y64"][m, n]) <= 1e-12 * out["absum"][m, n]
            assert out["y"][m, n] == np.float16(out["y64"][m, n])
    assert np.all(out["absum"] >= np.abs(out["y64"]))


# ------------------------------------------------- low-rank residual (plain SVD)
def _planted(n, m, s0, seed):
    rng = np.random.default_rng(seed)
    U0, _ = np.linalg.qr(rng.standard_normal((n, len(s0))))
    V0, _ = np.linalg.qr(rng.standard_normal((m, len(s0))))
    return U0, V0, U0 @ np.diag(s0) @ V0.T


def test_lowrank_recovers_a_planted_spectrum():
    """Delta W built from orthonormal U0, V0 and known singular values: the
    rank-r factors must give back those values, the product U0_r S0_r V0_r^T,
    orthonormal rows of A and B^T B = S_r^2; the residual is the Eckart-Young
    optimum sum_{i>r} s_i^2 (computed from the planted values, not an SVD)."""
    s0 = np.array([5.0, 3.5, 2.0, 1.25, 0.5, 0.25, 0.125, 0.0625])
    U0, V0, dW = _planted(40, 56, s0, seed=60)
    for r in (1, 3, 5, 8):
        out = oracle.lowrank(dW, r)
        assert np.allclose(out["sigma"], s0[:r], rtol=1e-12, atol=0)
        want = U0[:, :r] @ np.diag(s0[:r]) @ V0[:, :r].T
        assert np.abs(out["B"] @ out["A"] - want).max() <= 1e-12
        assert np.abs(out["A"] @ out["A"].T - np.eye(r)).max() <= 1e-12
        assert np.abs(out["B"].T @ out["B"] - np.diag(s0[:r] ** 2)).max() <= 1e-11
        resid = np.sum((dW - out["B"] @ out["A"]) ** 2)
        assert abs(resid - np.sum(s0[r:] ** 2)) <= 1e-12 * np.sum(s0 ** 2)


def test_lowrank_rank_one_and_zero():
    """A rank-one error u v^T has sigma_1 = |u| |v| and nothing else; a zero
    error gives zero factors."""
    rng = np.random.default_rng(61)
    u, v = rng.standard_normal(30), rng.standard_normal(20)
    out = oracle.lowrank(np.outer(u, v), 2)
    assert abs(out["sigma"][0] - np.linalg.norm(u) * np.linalg.norm(v)) <= 1e-12 * out["sigma"][0]
    assert out["sigma"][1] <= 1e-12 * out["sigma"][0]
    assert np.abs(out["B"][:, :1] @ out["A"][:1] - np.outer(u, v)).max() <= 1e-12 * np.abs(np.outer(u, v)).max()
    z = oracle.lowrank(np.zeros((12, 9)), 3)
    assert np.all(z["sigma"] == 0) and np.all(z["B"] @ z["A"] == 0)


def test_quant_error_is_w_minus_w_hat_and_within_half_a_step():
    """Delta W is W - W_hat exactly; for min-max round-to-nearest (no solver
    iterations) every error is at most half a code step s/2, plus what the fp16
    storage of s and z adds (L half-spacings of s, half a spacing of z times s)
    and the fp16 rounding of W_hat (half a spacing of |W_hat|)."""
    N, K, g = 16, 256, 64
    W = synth.student_t_host((N, K), seed=62, stream=0).astype(np.float16)
    r = oracle.quantize(W, 3, g, iters=0)
    dW = oracle.quant_error(W, r["codes"], r["scale"], r["zero"], g)
    Wh = oracle.dequantize(r["codes"], r["scale"], r["zero"], g).reshape(N, K)
    assert np.array_equal(dW, W.astype(np.float64) - Wh.astype(np.float64))
    rep = lambda a: np.repeat(a.reshape(N, K // g), g, axis=1)
    s16, z16 = rep(r["scale"]), rep(r["zero"])
    s = s16.astype(np.float64)
    sp = lambda a: np.spacing(np.abs(a).astype(np.float16)).astype(np.float64)
    bound = s / 2 + 7 * sp(s16) / 2 + sp(z16) / 2 * s + sp(Wh) / 2
    assert np.all(np.abs(dW) <= bound)
    assert np.count_nonzero(oracle.quant_error(Wh, r["codes"], r["scale"], r["zero"], g)) == 0
