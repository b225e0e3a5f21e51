"""GPU parity of the low-rank residual of the quantization error (hqq_lowrank,
through the C ABI) against the oracle's truncated SVD of the exact Delta W.

Where sigma_r is well separated from sigma_{r+1} the rank-r factorization is
unique (up to signs) and the randomized subspace iteration converges to it:
there the singular values and B A are compared with the oracle's (relative
tolerance 1e-4 of sigma_1: fp32 products over K terms, fp32 storage of the
sketch).  On the nearly flat spectrum of a real quantization error the rank-r
subspace is not well determined, so properties that hold for any sketch are
checked: estimates never exceed the exact values (Ritz values of a subspace),
they capture most of the optimal energy, A has orthonormal rows, and
||Delta W - B A||_F^2 = ||Delta W||_F^2 - sum sigma^2 >= the Eckart-Young
optimum."""
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


def _setup(hqq, W0, nbits, group, iters=2):
    rows, cols = W0.shape
    r = oracle.quantize(W0, nbits, group, iters=iters)
    q = hqq.QuantizedMatrix(torch.from_numpy(r["packed"]).cuda(),
                            torch.from_numpy(r["scale"].reshape(rows, cols // group)).cuda(),
                            torch.from_numpy(r["zero"].reshape(rows, cols // group)).cuda(),
                            rows, cols, nbits, group)
    Wh = oracle.dequantize(r["codes"], r["scale"], r["zero"], group).reshape(rows, cols)
    return q, r, Wh


def _omega(cols, sketch, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.standard_normal((cols, sketch)).astype(np.float32)).cuda()


def _run(hqq, W, q, rank, sketch, iters, seed=7):
    B, A, s = hqq.hqq_lowrank(torch.from_numpy(W).cuda(), q, rank, _omega(q.cols, sketch, seed),
                              power_iters=iters)
    torch.cuda.synchronize()
    return B.cpu().numpy().astype(np.float64), A.cpu().numpy().astype(np.float64), \
        s.cpu().numpy().astype(np.float64)


def _planted_w(Wh, rank, scale, seed):
    """W = fp16(W_hat + D) with D of `rank` planted singular values in [scale/2, scale]."""
    rows, cols = Wh.shape
    rng = np.random.default_rng(seed)
    U0, _ = np.linalg.qr(rng.standard_normal((rows, rank)))
    V0, _ = np.linalg.qr(rng.standard_normal((cols, rank)))
    D = U0 @ np.diag(np.linspace(scale, scale / 2, rank)) @ V0.T
    return (Wh.astype(np.float64) + D).astype(np.float16)


@pytest.mark.parametrize("nbits,group,rows,cols,rank,sketch", [
    (4, 64, 200, 320, 8, 16), (3, 64, 256, 512, 8, 32), (2, 16, 130, 96, 5, 16),
    (8, 128, 96, 256, 12, 32), (1, 32, 300, 192, 16, 64), (3, 128, 520, 1024, 24, 64)])
def test_lowrank_planted_gap_matches_the_svd(hqq, nbits, group, rows, cols, rank, sketch):
    W0 = synth.student_t_host((rows, cols), seed=70, stream=rows + nbits).astype(np.float16)
    q, r, Wh = _setup(hqq, W0, nbits, group)
    W = _planted_w(Wh, rank, scale=4.0, seed=rows)
    dW = oracle.quant_error(W, r["codes"], r["scale"], r["zero"], group)
    ref = oracle.lowrank(dW, rank)
    assert ref["sigma_all"][rank] < 0.05 * ref["sigma"][-1]           # the planted gap
    B, A, s = _run(hqq, W, q, rank, sketch, iters=2)
    s1 = ref["sigma"][0]
    assert np.abs(s - ref["sigma"]).max() <= 1e-4 * s1, (s, ref["sigma"])
    BA, BA_ref = B @ A, ref["B"] @ ref["A"]
    assert np.abs(BA - BA_ref).max() <= 1e-4 * np.abs(BA_ref).max() + 1e-4 * ref["sigma_all"][rank]
    assert np.abs(A @ A.T - np.eye(rank)).max() <= 1e-4


@pytest.mark.parametrize("nbits,group,rows,cols,rank,sketch,iters", [
    (3, 64, 384, 512, 16, 32, 2), (4, 64, 256, 256, 8, 16, 2), (2, 32, 512, 384, 32, 64, 3)])
def test_lowrank_flat_spectrum_properties(hqq, nbits, group, rows, cols, rank, sketch, iters):
    W = synth.student_t_host((rows, cols), seed=71, stream=rows).astype(np.float16)
    q, r, Wh = _setup(hqq, W, nbits, group)
    dW = oracle.quant_error(W, r["codes"], r["scale"], r["zero"], group)
    ref = oracle.lowrank(dW, rank)
    B, A, s = _run(hqq, W, q, rank, sketch, iters)
    assert np.all(np.diff(s) <= 1e-6 * s[0])                           # decreasing
    assert np.all(s <= ref["sigma"] * (1 + 1e-4))                       # Ritz values
    assert np.sum(s ** 2) >= 0.8 * np.sum(ref["sigma"] ** 2)
    assert np.abs(A @ A.T - np.eye(rank)).max() <= 1e-4
    total = np.sum(dW ** 2)
    resid = np.sum((dW - B @ A) ** 2)
    assert abs(resid - (total - np.sum(s ** 2))) <= 1e-4 * total
    assert resid >= (total - np.sum(ref["sigma"] ** 2)) * (1 - 1e-4)


def test_lowrank_zero_and_rank_deficient_errors(hqq):
    rows, cols, group = 128, 256, 64
    W0 = synth.student_t_host((rows, cols), seed=72, stream=0).astype(np.float16)
    q, r, Wh = _setup(hqq, W0, 4, group)
    B, A, s = _run(hqq, Wh, q, 4, 16, 2)                 # W = W_hat exactly: no error
    assert np.all(B == 0) and np.all(A == 0) and np.all(s == 0)
    W = _planted_w(Wh, 3, scale=2.0, seed=3)              # error of rank 3 (+ fp16 rounding)
    dW = oracle.quant_error(W, r["codes"], r["scale"], r["zero"], group)
    ref = oracle.lowrank(dW, 6)
    B, A, s = _run(hqq, W, q, 6, 16, 2)
    assert np.abs(s[:3] - ref["sigma"][:3]).max() <= 1e-4 * ref["sigma"][0]
    assert np.all(s[3:] <= 1e-3 * s[0])            # what is left is fp16 rounding noise
    top, top_ref = B[:, :3] @ A[:3], ref["B"][:, :3] @ ref["A"][:3]    # unique: the planted part
    assert np.abs(top - top_ref).max() <= 1e-4 * np.abs(top_ref).max() + 1e-4 * ref["sigma"][3]


def test_lowrank_full_size_gate_properties(hqq):
    """The 28672 x 8192 3-bit g64 matrix, rank 16 from a 32-column sketch:
    orthonormal A, decreasing sigma, and the residual identity, with Delta W
    and the residual formed on the GPU in fp64."""
    rows, cols, group = 28672, 8192, 64
    Wd = synth.student_t_device((rows, cols), seed=5, stream=4)
    q = hqq.hqq_quantize(Wd, nbits=3, group=group)
    om = _omega(cols, 32, 11)
    B, A, s = hqq.hqq_lowrank(Wd, q, 16, om, power_iters=2)
    dW = Wd.double() - hqq.hqq_dequantize(q).double()
    total = float((dW ** 2).sum())
    resid = float(((dW - B.double() @ A.double()) ** 2).sum())
    s64 = s.double()
    assert bool((s64[1:] <= s64[:-1] * (1 + 1e-6)).all())
    eye = A.double() @ A.double().T
    assert float((eye - torch.eye(16, dtype=torch.float64, device=eye.device)).abs().max()) <= 1e-4
    assert abs(resid - (total - float((s64 ** 2).sum()))) <= 1e-4 * total
    assert float(s64[0]) > 0
