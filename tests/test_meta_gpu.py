"""GPU parity of the 8-bit meta data (section 4.1 of the HQQ page: zero points
in 8 bits without grouping, scales in 8 bits in groups of 128) through the C
ABI, against the CPU oracle on the same inputs.

Tolerance: everything is integer or the same binary32 sequence on both sides,
so codes and the fp16 second-level scales and restored values must be
identical bit for bit, and the second-level zeros equal in value (the sign of
a zero z is not specified: -0 and +0 restore identically).
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def hqq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import weight_only_quantization_b200 as m
    return m


def _meta_of_matrix(hqq, shape, nbits, group, seed, stream=0):
    W = synth.student_t_device(shape, seed=seed, stream=stream)
    q = hqq.hqq_quantize(W, nbits=nbits, group=group)
    torch.cuda.synchronize()
    return q


def _check_meta(hqq, x_dev, mgroup, label):
    m = hqq.hqq_meta_quantize(x_dev.reshape(-1), mgroup)
    torch.cuda.synchronize()
    x = x_dev.reshape(-1).cpu().numpy()
    ref = oracle.meta_quantize(x, mgroup)
    codes = m.codes.cpu().numpy()
    sc = m.scale.cpu().numpy()
    ze = m.zero.cpu().numpy()
    assert np.array_equal(codes, ref["codes"]), (label, int(np.sum(codes != ref["codes"])))
    assert np.array_equal(sc.view(np.uint16), ref["scale"].view(np.uint16)), label
    assert np.array_equal(ze.astype(np.float32), ref["zero"].astype(np.float32)), label
    back = hqq.hqq_meta_dequantize(m)
    torch.cuda.synchronize()
    want = oracle.meta_dequantize(ref["codes"], ref["scale"], ref["zero"], mgroup)
    assert np.array_equal(back.cpu().numpy().view(np.uint16), want.view(np.uint16)), label
    return m, ref


@pytest.mark.parametrize("which", ["zero", "scale"])
@pytest.mark.parametrize("mgroup", [0, 128, 1, 2, 16, 32, 64, 4096])
def test_meta_of_a_quantized_matrix(hqq, which, mgroup):
    q = _meta_of_matrix(hqq, (512, 2048), 3, 64, seed=31)
    _check_meta(hqq, getattr(q, which), mgroup, f"{which} g{mgroup}")


@pytest.mark.parametrize("n", [1, 2, 7, 8, 9, 100, 1000, 4095, 4096, 4097, 5003, 65536 + 3])
@pytest.mark.parametrize("mgroup", [0, 128])
def test_meta_ragged_lengths(hqq, n, mgroup):
    """Lengths around the vector width (8), the warp (32), the small/cluster
    switch of one-group tensors (4096) and ragged last groups."""
    rng = np.random.default_rng(n)
    x = torch.from_numpy(rng.uniform(-3, 12, n).astype(np.float16)).cuda()
    _check_meta(hqq, x, mgroup, f"n={n} g{mgroup}")


def test_meta_empty(hqq):
    x = torch.empty(0, dtype=torch.float16, device="cuda")
    m = hqq.hqq_meta_quantize(x, 0)
    assert m.codes.numel() == 0 and m.scale.numel() == 0


@pytest.mark.parametrize("case", ["constant", "signed_zeros", "two_levels", "fp16_extremes",
                                  "tiny_range", "subnormals"])
def test_meta_degenerate_inputs(hqq, case):
    n = 12345
    rng = np.random.default_rng(7)
    if case == "constant":
        x = np.full(n, 3.25, np.float16)
    elif case == "signed_zeros":
        x = np.where(rng.random(n) < 0.5, np.float16(0.0), np.float16(-0.0)).astype(np.float16)
        x[::97] = np.float16(1.5)
    elif case == "two_levels":
        x = np.where(rng.random(n) < 0.5, np.float16(-2.0), np.float16(5.0)).astype(np.float16)
    elif case == "fp16_extremes":
        x = rng.uniform(-1, 1, n).astype(np.float16)
        x[5], x[900] = np.float16(-65504.0), np.float16(65504.0)
    elif case == "tiny_range":
        x = (np.float16(7.0) + rng.integers(0, 3, n).astype(np.float16) * np.float16(2 ** -8))
        x = x.astype(np.float16)
    else:
        x = (rng.integers(-40, 40, n) * 2.0 ** -24).astype(np.float16)
    xd = torch.from_numpy(x).cuda()
    for mg in (0, 128, 1):
        _check_meta(hqq, xd, mg, f"{case} g{mg}")


@pytest.mark.parametrize("nbits,group", [(4, 64), (3, 64), (2, 32), (2, 16), (4, 128)])
@pytest.mark.parametrize("scale_8bit", [False, True])
def test_dequantize_with_8bit_meta(hqq, nbits, group, scale_8bit):
    """One-pass weight dequantization from 8-bit zero points (one group) and
    fp16 or 8-bit (groups of 128) scales equals, bit for bit, the oracle's
    restore-then-dequantize."""
    rows, cols = 77, 10 * group
    q = _meta_of_matrix(hqq, (rows, cols), nbits, group, seed=32, stream=nbits)
    zq = hqq.hqq_meta_quantize(q.zero.reshape(-1), 0)
    sq = hqq.hqq_meta_quantize(q.scale.reshape(-1), 128) if scale_8bit else None
    out = hqq.hqq_dequantize_meta(q.packed, zq, rows, cols, nbits, group,
                                  scale=None if scale_8bit else q.scale, scale_q=sq)
    torch.cuda.synchronize()
    codes = oracle.unpack(q.packed.cpu().numpy(), rows * cols, nbits)
    zdict = dict(codes=zq.codes.cpu().numpy(), scale=zq.scale.cpu().numpy(),
                 zero=zq.zero.cpu().numpy())
    if scale_8bit:
        sdict = dict(codes=sq.codes.cpu().numpy(), scale=sq.scale.cpu().numpy(),
                     zero=sq.zero.cpu().numpy())
        want = oracle.dequantize_meta(codes, group, zdict, 0, scale_q=sdict, scale_group=128)
    else:
        want = oracle.dequantize_meta(codes, group, zdict, 0,
                                      scale=q.scale.cpu().numpy().reshape(-1))
    assert np.array_equal(out.cpu().numpy().reshape(-1).view(np.uint16), want.view(np.uint16))
    # and the fused pass equals the two-step form of the library itself
    z16 = hqq.hqq_meta_dequantize(zq).reshape(q.zero.shape)
    s16 = hqq.hqq_meta_dequantize(sq).reshape(q.scale.shape) if scale_8bit else q.scale
    two = hqq.hqq_dequantize(hqq.QuantizedMatrix(q.packed, s16, z16, rows, cols, nbits, group))
    torch.cuda.synchronize()
    assert torch.equal(two.view(torch.int16), out.view(torch.int16))


def test_full_size_zero_points_of_the_70b_gate_matrix(hqq):
    """The whole-tensor (cluster) path on the zero points of a 28672 x 8192
    3-bit g64 matrix (3.67 M values), and the one-pass dequantization from them,
    checked on sampled rows."""
    rows, cols, nbits, group = 28672, 8192, 3, 64
    q = _meta_of_matrix(hqq, (rows, cols), nbits, group, seed=5, stream=4)
    m, ref = _check_meta(hqq, q.zero, 0, "70b gate zero")
    sq, _ = _check_meta(hqq, q.scale, 128, "70b gate scale")
    out = hqq.hqq_dequantize_meta(q.packed, m, rows, cols, nbits, group, scale_q=sq)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    pk = q.packed.cpu().numpy()
    z16 = oracle.meta_dequantize(ref["codes"], ref["scale"], ref["zero"], 0)
    s_all = oracle.meta_dequantize(sq.codes.cpu().numpy(), sq.scale.cpu().numpy(),
                                   sq.zero.cpu().numpy(), 128)
    codes = oracle.unpack(pk, rows * cols, nbits)
    for r in rng.choice(rows, 24, replace=False):
        sl = slice(r * cols, (r + 1) * cols)
        gs = slice(r * cols // group, (r + 1) * cols // group)
        want = oracle.dequantize(codes[sl], s_all[gs], z16[gs], group)
        got = out[r].cpu().numpy()
        assert np.array_equal(got.view(np.uint16), want.view(np.uint16)), r


def test_meta_bad_arguments(hqq):
    x = torch.zeros(100, dtype=torch.float16, device="cuda")
    with pytest.raises(hqq.HQQError):
        hqq.hqq_meta_quantize(x, 100)
    with pytest.raises(hqq.HQQError):
        hqq.hqq_meta_quantize(x[1:], 0)          # 16-byte alignment of x
    m = hqq.hqq_meta_quantize(x, 0)
    with pytest.raises(hqq.HQQError):
        hqq.hqq_dequantize_meta(torch.zeros(32, dtype=torch.uint8, device="cuda"), m, 1, 64, 4,
                                64, scale=torch.zeros(1, dtype=torch.float16, device="cuda"),
                                scale_q=m)


def test_meta_quantize_batch_matches_oracle_and_single_calls(hqq):
    """One batch of whole-tensor and grouped meta tensors (ragged, tiny, empty,
    more than one launch's worth) equals the oracle and the per-tensor calls
    bit for bit."""
    rng = np.random.default_rng(31)
    specs = []
    for i in range(150):                      # > 128 tensors: several launches
        n = int(rng.choice([0, 1, 7, 100, 1000, 4099, 70001, 262144]))
        mg = int(rng.choice([0, 0, 1, 8, 128, 256, 1 << 20]))
        specs.append((n, mg))
    xs = []
    for i, (n, mg) in enumerate(specs):
        x = (rng.standard_normal(n) * (1 + i % 5) + i % 3).astype(np.float16)
        xs.append(x)
    dev = [torch.from_numpy(x).cuda() for x in xs]
    got = hqq.hqq_meta_quantize_batch([(d, mg) for d, (n, mg) in zip(dev, specs)])
    single = [hqq.hqq_meta_quantize(d, mg) if d.numel() else None
              for d, (n, mg) in zip(dev, specs)]
    torch.cuda.synchronize()
    for x, (n, mg), m, one in zip(xs, specs, got, single):
        ref = oracle.meta_quantize(x, mg)
        assert np.array_equal(m.codes.cpu().numpy(), ref["codes"]), (n, mg)
        assert np.array_equal(m.scale.cpu().numpy().view(np.uint16), ref["scale"].view(np.uint16))
        assert np.array_equal(m.zero.cpu().numpy().view(np.uint16), ref["zero"].view(np.uint16))
        if one is not None:
            assert torch.equal(one.codes, m.codes) and torch.equal(one.zero, m.zero)


def test_meta_quantize_batch_bad_job_launches_nothing(hqq):
    x = torch.zeros(64, dtype=torch.float16, device="cuda")
    good = hqq.Meta8(torch.full((64,), 7, dtype=torch.uint8, device="cuda"),
                     torch.zeros(1, dtype=torch.float16, device="cuda"),
                     torch.zeros(1, dtype=torch.float16, device="cuda"), 0)
    with pytest.raises(hqq.HQQError):
        hqq.hqq_meta_quantize_batch([(x, 0), (x, 3)], outputs=[good, good])   # 3: not 2^k
    torch.cuda.synchronize()
    assert torch.all(good.codes == 7)
