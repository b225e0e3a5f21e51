"""GPU parity of the weight-only linear layer (hqq_linear, through the C ABI):
Y = X W_hat^T with W_hat the dequantized fp16 weights, against the oracle's
fp64 product on the oracle's own quantization of the same weights.

Tolerance (from the arithmetic of both kernels): every product of two fp16
values is exact in fp32, and the kernels add them in fp32 along chains of
bounded length -- the tensor-core kernel accumulates ceil(K/16) MMAs of 16
products each in tensor memory, then adds at most 8 split-k partials; the
few-token kernel accumulates each warp's 16-wide k steps, then the 8 warps'
sums and at most 8 cluster ranks' sums.  No product passes through more than
D = ceil(K/16) + 40 additions (16 products inside one MMA: at most 5 levels),
so with u = 2^-23 (one unit of an fp32 add, truncating or rounding) and
S = sum_k |x_k w_k| the fp32 result is within 1.001 D u S of the exact sum
(first-order bound of any summation tree of depth D); one fp16 rounding adds
2^-11 of the value and at most 2^-25 near zero:
    |Y_gpu - Y_exact| <= 2^-11 |Y_exact| + 1.001 D 2^-23 S + 2^-24.
At K = 8192 this is 6.6e-5 S, where one group of 64 weights with a wrong
scale or code offset moves an output by about 8 |x| |w| -- some 20x the
bound on the synthetic weights, so such a defect cannot hide in it.  On small
integer data every partial sum is an integer below 2^24 and the result must
equal the exact one rounded to fp16 (tested up to K = 28672).
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


def _depth(K):
    """Longest chain of fp32 additions any product passes through."""
    return -(-K // 16) + 40


def _check(Y_gpu, X, Wh, label):
    ref = oracle.linear(X, Wh)
    K = X.shape[1]
    y = Y_gpu.astype(np.float64)
    tol = 2.0 ** -11 * np.abs(ref["y64"]) + 1.001 * _depth(K) * 2.0 ** -23 * ref["absum"] \
        + 2.0 ** -24
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


def _integer_matrix(hqq, rows, cols, nbits, group, seed):
    """A quantized matrix whose W_hat is exact on small numbers: random codes,
    per-group scales in {1/2, 1, 2} and integer zero points in [0, L], packed
    by the oracle.  W_hat = (c - z) s is a multiple of 1/2 with |W_hat| <= 2L,
    so any wrong scale or zero of a group changes the exact product."""
    L = (1 << nbits) - 1
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, L + 1, rows * cols).astype(np.uint8)
    ng = rows * cols // group
    scale = rng.choice(np.array([0.5, 1.0, 2.0], np.float16), ng)
    zero = rng.integers(0, L + 1, ng).astype(np.float16)
    q = hqq.QuantizedMatrix(torch.from_numpy(oracle.pack(codes, nbits)).cuda(),
                            torch.from_numpy(scale.reshape(rows, cols // group)).cuda(),
                            torch.from_numpy(zero.reshape(rows, cols // group)).cuda(),
                            rows, cols, nbits, group)
    Wh = oracle.dequantize(codes, scale, zero, group).reshape(rows, cols)
    return q, Wh


@pytest.mark.parametrize("rows,cols", [(200, 8192), (130, 28672)])
@pytest.mark.parametrize("nbits", [3, 4])
@pytest.mark.parametrize("M", [1, 8, 16, 17, 32, 256, 1030, 2048])
def test_linear_exact_full_size_k(hqq, rows, cols, nbits, M):
    """Bit-exact at the 70B shapes' input sizes (K = 8192 and 28672): with
    |x| <= 4 and |W_hat| <= 30 in steps of 1/2, every partial sum of any order
    is a multiple of 1/2 below 2^23 in magnitude, hence exact in fp32, so Y
    must equal the exact product rounded once to fp16.  Rows off the 128-row
    tile; token counts covering the few-token kernel (1-16 tokens, clusters
    splitting k), the tensor-memory kernel's small tiles with split-k
    clusters (17, 32), its 256-token tiles and its 512-token tiles (1030,
    2048)."""
    q, Wh = _integer_matrix(hqq, rows, cols, nbits, 64, seed=rows + nbits)
    rng = np.random.default_rng(M + cols)
    X = rng.integers(-4, 5, (M, cols)).astype(np.float16)
    Y = hqq.hqq_linear(torch.from_numpy(X).cuda(), q)
    torch.cuda.synchronize()
    ref = oracle.linear(X, Wh)
    assert np.abs(ref["absum"]).max() < 2.0 ** 23
    got = Y.cpu().numpy()
    bad = got.view(np.uint16) != ref["y"].view(np.uint16)
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5].tolist())


@pytest.mark.parametrize("nbits,group", [(3, 64), (3, 32), (3, 16), (4, 64), (2, 16), (8, 32), (1, 128)])
@pytest.mark.parametrize("M", [4, 8, 9, 15, 16, 24, 32, 33])
def test_linear_decode_token_blocks(hqq, nbits, group, M):
    """Token counts inside and at the edges of the few-token kernel's 8-token
    MMA column blocks (1, 2 and 4 blocks) and the first count past them; at 3
    bits, 9 to 16 tokens take the kernel whose CTAs share one staged copy of X
    (200 features: a partly empty 128-feature CTA tile)."""
    rows, cols = 200, 1024
    W = synth.student_t_host((rows, cols), seed=53, stream=nbits * 1000 + M).astype(np.float16)
    q, Wh, _ = _quantized(hqq, W, nbits, group)
    X = _tokens(M, cols, seed=M + 7)
    Y = hqq.hqq_linear(torch.from_numpy(X).cuda(), q)
    torch.cuda.synchronize()
    _check(Y.cpu().numpy(), X, Wh, f"{nbits}b g{group} M={M}")


@pytest.mark.parametrize("nbits,group,rows,cols", [(3, 64, 130, 1088), (4, 16, 48, 16384),
                                                   (1, 32, 77, 96), (8, 64, 33, 512)])
@pytest.mark.parametrize("M", [1, 5, 8, 12])
def test_linear_decode_packed_alignment(hqq, nbits, group, rows, cols, M):
    """A packed buffer that is 4-byte but not 16-byte aligned takes the
    few-token kernels' direct-load form; it must give the same bits as the
    staged form on an aligned copy (same products, same summation order).  At
    3 bits, 8 and 12 tokens take the kernel whose CTAs share a staged X; past
    8 tokens the other widths take the many-token kernel for both copies."""
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


@pytest.mark.parametrize("shape,stream", [((28672, 8192), 4), ((8192, 28672), 6)])
@pytest.mark.parametrize("M", [1, 16, 256, 2048])
def test_linear_full_size_70b_gate_sampled(hqq, M, shape, stream):
    """The 28672 x 8192 gate and 8192 x 28672 down matrices (3-bit g64)
    quantized on the GPU; sampled output features checked against the
    oracle's own quantization of those rows (whose codes, scales and zeros
    must equal the GPU's)."""
    (rows, cols), nbits, group = shape, 3, 64
    W = synth.student_t_device((rows, cols), seed=5, stream=stream)
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
    _check(Y.cpu().numpy()[:, sample], X, Wh, f"70b {rows}x{cols} M={M}")


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
