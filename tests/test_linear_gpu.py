"""GPU parity of the weight-only linear layer (hqq_linear, through the C ABI):
Y = X W_hat^T with W_hat the dequantized fp16 weights, against the oracle's
fp64 product on the oracle's own quantization of the same weights.

Tolerance (from the arithmetic): the kernel forms the products of fp16 values
exactly and sums them in fp32 in an unspecified order, then rounds to fp16.
With S = sum_k |x_k w_k| and g = K * 2^-23 (a generous bound on the relative
accumulation error of K fp32 additions, tensor-core internal rounding
included):  |Y_gpu - Y_exact| <= 2^-11 |Y_exact| + 2 g S + 2^-24.
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


def _quantized(hqq, W, nbits, group, iters=2):
    """Oracle quantization of W, uploaded as a QuantizedMatrix."""
    r = oracle.quantize(W, nbits, group, iters=iters)
    rows, cols = W.shape
    q = hqq.QuantizedMatrix(torch.from_numpy(r["packed"]).cuda(),
                            torch.from_numpy(r["scale"].reshape(rows, cols // group)).cuda(),
                            torch.from_numpy(r["zero"].reshape(rows, cols // group)).cuda(),
                            rows, cols, nbits, group)
    Wh = oracle.dequantize(r["codes"], r["scale"], r["zero"], group).reshape(rows, cols)
    return q, Wh, r


def _tokens(M, K, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((M, K)).astype(np.float16)


def _check(Y_gpu, X, Wh, label):
    ref = oracle.linear(X, Wh)
    K = X.shape[1]
    y = Y_gpu.astype(np.float64)
    tol = 2.0 ** -11 * np.abs(ref["y64"]) + 2 * K * 2.0 ** -23 * ref["absum"] + 2.0 ** -24
    err = np.abs(y - ref["y64"])
    bad = err > tol
    assert not bad.any(), (label, int(bad.sum()), float((err / tol).max()))
    return float((err / tol).max())


@pytest.mark.parametrize("nbits,group", [(4, 64), (3, 64), (2, 32), (4, 128), (2, 16), (3, 256),
                                         (8, 128), (1, 64)])
@pytest.mark.parametrize("M", [1, 2, 3, 16, 100, 256])
def test_linear_formats_and_token_counts(hqq, nbits, group, M):
    rows, cols = 256, 1024
    W = synth.student_t_host((rows, cols), seed=50, stream=nbits * 100 + group).astype(np.float16)
    q, Wh, _ = _quantized(hqq, W, nbits, group)
    X = _tokens(M, cols, seed=M)
    Y = hqq.hqq_linear(torch.from_numpy(X).cuda(), q)
    torch.cuda.synchronize()
    _check(Y.cpu().numpy(), X, Wh, f"{nbits}b g{group} M={M}")


@pytest.mark.parametrize("rows,cols,M", [(128, 64, 1), (300, 192, 17), (129, 320, 33), (77, 48, 2),
                                         (130, 8208, 1), (200, 512, 1030), (256, 1024, 2048),
                                         (1000, 2048, 300), (64, 4096, 513), (384, 16, 7),
                                         (200, 8208, 65)])
def test_linear_ragged_shapes(hqq, rows, cols, M):
    """Feature counts off the 128-row tile, input sizes off the 64-wide k-tile
    (down to one group of 16) and longer than the stage ring, token counts off
    every token tile."""
    group = 16 if cols % 64 else 64
    nbits = 3
    W = synth.student_t_host((rows, cols), seed=51, stream=rows).astype(np.float16)
    q, Wh, _ = _quantized(hqq, W, nbits, group)
    X = _tokens(M, cols, seed=rows + M)
    Y = hqq.hqq_linear(torch.from_numpy(X).cuda(), q)
    torch.cuda.synchronize()
    _check(Y.cpu().numpy(), X, Wh, f"{rows}x{cols} M={M}")


def test_linear_status_and_empty(hqq):
    rows, cols = 128, 256
    W = synth.student_t_host((rows, cols), seed=52, stream=0).astype(np.float16)
    q, Wh, _ = _quantized(hqq, W, 4, 64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    X = _tokens(40, cols, seed=1)
    Y = hqq.hqq_linear(torch.from_numpy(X).cuda(), q, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check(Y.cpu().numpy(), X, Wh, "status")
    E = hqq.hqq_linear(torch.zeros((0, cols), dtype=torch.float16, device="cuda"), q)
    assert E.shape == (0, rows)


@pytest.mark.parametrize("M", [1, 8, 32, 96])
def test_linear_exact_on_integer_data(hqq, M):
    """Small integers keep every product and partial sum exact in fp32, so the
    result must equal the exact one rounded to fp16, whatever the order (the
    few-token kernel's 8-token blocks at 1, 8 and 32 tokens; tensor-memory
    tiles at 96)."""
    rows, cols, group = 256, 512, 64
    rng = np.random.default_rng(9)
    W = rng.integers(-8, 8, (rows, cols)).astype(np.float16)
    W[:, 0::group] = -8                     # every group spans [-8, 7]: s = 1, z = 8
    W[:, 1::group] = 7
    q, Wh, r = _quantized(hqq, W, 4, group, iters=0)
    assert np.array_equal(Wh.astype(np.float32), W.astype(np.float32))
    X = rng.integers(-4, 5, (M, cols)).astype(np.float16)
    Y = hqq.hqq_linear(torch.from_numpy(X).cuda(), q)
    torch.cuda.synchronize()
    ref = oracle.linear(X, Wh)
    assert np.array_equal(Y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("nbits,group", [(3, 64), (4, 64), (2, 16), (8, 32), (1, 128)])
@pytest.mark.parametrize("M", [4, 8, 9, 15, 24, 32, 33])
def test_linear_decode_token_blocks(hqq, nbits, group, M):
    """Token counts inside and at the edges of the few-token kernel's 8-token
    MMA column blocks (1, 2 and 4 blocks) and the first count past them."""
    rows, cols = 200, 1024
    W = synth.student_t_host((rows, cols), seed=53, stream=nbits * 1000 + M).astype(np.float16)
    q, Wh, _ = _quantized(hqq, W, nbits, group)
    X = _tokens(M, cols, seed=M + 7)
    Y = hqq.hqq_linear(torch.from_numpy(X).cuda(), q)
    torch.cuda.synchronize()
    _check(Y.cpu().numpy(), X, Wh, f"{nbits}b g{group} M={M}")


@pytest.mark.parametrize("nbits,group,rows,cols", [(3, 64, 130, 1088), (4, 16, 48, 16384),
                                                   (1, 32, 77, 96), (8, 64, 33, 512)])
@pytest.mark.parametrize("M", [1, 5])
def test_linear_decode_packed_alignment(hqq, nbits, group, rows, cols, M):
    """A packed buffer that is 4-byte but not 16-byte aligned takes the
    few-token kernel's direct-load form; it must give the same bits as the
    staged form on an aligned copy (same products, same summation order)."""
    W = synth.student_t_host((rows, cols), seed=54, stream=rows + nbits).astype(np.float16)
    q, Wh, r = _quantized(hqq, W, nbits, group)
    shift = 8 if nbits == 8 else 4
    raw = torch.zeros(q.packed.numel() + 16, dtype=torch.uint8, device="cuda")
    base = (16 - raw.data_ptr() % 16) % 16
    un = raw[base + shift: base + shift + q.packed.numel()]
    un.copy_(q.packed)
    assert un.data_ptr() % 16 == shift
    qu = hqq.QuantizedMatrix(un, q.scale, q.zero, rows, cols, nbits, group)
    X = torch.from_numpy(_tokens(M, cols, seed=rows + M)).cuda()
    Ya = hqq.hqq_linear(X, q)
    Yu = hqq.hqq_linear(X, qu)
    torch.cuda.synchronize()
    assert torch.equal(Ya, Yu)
    _check(Yu.cpu().numpy(), X.cpu().numpy(), Wh, f"unaligned {nbits}b M={M}")


@pytest.mark.parametrize("M", [1, 16, 256, 2048])
def test_linear_full_size_70b_gate_sampled(hqq, M):
    """The 28672 x 8192 3-bit g64 gate matrix quantized on the GPU; sampled
    output features checked against the oracle's own quantization of those
    rows (whose codes, scales and zeros must equal the GPU's)."""
    rows, cols, nbits, group = 28672, 8192, 3, 64
    W = synth.student_t_device((rows, cols), seed=5, stream=4)
    q = hqq.hqq_quantize(W, nbits=nbits, group=group)
    X = _tokens(M, cols, seed=77)
    Y = hqq.hqq_linear(torch.from_numpy(X).cuda(), q)
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    sample = np.sort(rng.choice(rows, 40, replace=False))
    Wn = W[torch.from_numpy(sample).cuda()].cpu().numpy()
    r = oracle.quantize(Wn, nbits, group)
    gs = cols // group
    sc = q.scale.view(-1).cpu().numpy().reshape(rows, gs)[sample].reshape(-1)
    ze = q.zero.view(-1).cpu().numpy().reshape(rows, gs)[sample].reshape(-1)
    assert np.array_equal(sc.view(np.uint16), r["scale"].view(np.uint16))
    assert np.array_equal(ze.astype(np.float32), r["zero"].astype(np.float32))
    codes_all = oracle.unpack(q.packed.cpu().numpy(), rows * cols, nbits).reshape(rows, cols)
    assert np.array_equal(codes_all[sample].reshape(-1), r["codes"])
    Wh = oracle.dequantize(r["codes"], r["scale"], r["zero"], group).reshape(len(sample), cols)
    _check(Y.cpu().numpy()[:, sample], X, Wh, f"70b gate M={M}")


def test_linear_bad_arguments(hqq):
    rows, cols = 128, 256
    W = synth.student_t_host((rows, cols), seed=53, stream=0).astype(np.float16)
    q, _, _ = _quantized(hqq, W, 4, 64)
    X = torch.zeros((4, cols + 8), dtype=torch.float16, device="cuda")
    with pytest.raises(ValueError):
        hqq.hqq_linear(X, q)                           # wrong inner size
    Xm = torch.zeros((4, cols + 8), dtype=torch.float16, device="cuda")[:, 1:cols + 1]
    with pytest.raises(ValueError):
        hqq.hqq_linear(Xm, q)                          # not contiguous
    L = hqq._lib
    P = lambda t: None if t is None else __import__("ctypes").c_void_p(t)
    Xd = torch.zeros((4, cols), dtype=torch.float16, device="cuda")
    Yd = torch.zeros((4, rows), dtype=torch.float16, device="cuda")
    st = L.hqq_linear(P(Xd.data_ptr() + 2), 4, P(q.packed.data_ptr()), P(q.scale.data_ptr()),
                      P(q.zero.data_ptr()), rows, cols, 4, 64, P(Yd.data_ptr()), None, None)
    assert st == 5                                      # X not 16-byte aligned
    st = L.hqq_linear(P(Xd.data_ptr()), -1, P(q.packed.data_ptr()), P(q.scale.data_ptr()),
                      P(q.zero.data_ptr()), rows, cols, 4, 64, P(Yd.data_ptr()), None, None)
    assert st == 2


@pytest.mark.parametrize("nbits,group", [(3, 64), (4, 64), (2, 16), (8, 128)])
@pytest.mark.parametrize("M", [1, 3, 100, 1030])
@pytest.mark.parametrize("scale_8bit", [False, True])
def test_linear_with_8bit_meta(hqq, nbits, group, M, scale_8bit):
    """Zero points (one group) and optionally scales (groups of 128) in their
    8-bit form, restored inside the kernel: against the oracle's restore, Q^-1
    and fp64 product (all inputs quantized by the oracle)."""
    rows, cols = 200, 8 * group
    W = synth.student_t_host((rows, cols), seed=60, stream=nbits * 10 + group).astype(np.float16)
    q, _, r = _quantized(hqq, W, nbits, group)
    zq = oracle.meta_quantize(r["zero"], 0)
    sq = oracle.meta_quantize(r["scale"], 128) if scale_8bit else None
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    zq8 = hqq.Meta8(dev(zq["codes"]), dev(zq["scale"]), dev(zq["zero"]), 0)
    sq8 = hqq.Meta8(dev(sq["codes"]), dev(sq["scale"]), dev(sq["zero"]), 128) if scale_8bit else None
    X = _tokens(M, cols, seed=M + 5)
    Y = hqq.hqq_linear_meta(torch.from_numpy(X).cuda(), q.packed, zq8, rows, cols, nbits, group,
                            scale=None if scale_8bit else q.scale, scale_q=sq8)
    torch.cuda.synchronize()
    if scale_8bit:
        Wh = oracle.dequantize_meta(r["codes"], group, zq, 0, scale_q=sq, scale_group=128)
    else:
        Wh = oracle.dequantize_meta(r["codes"], group, zq, 0, scale=r["scale"])
    _check(Y.cpu().numpy(), X, Wh.reshape(rows, cols), f"meta {nbits}b g{group} M={M}")
