"""The seeded input generator: Philox4x32-10 and the weight distribution."""
import numpy as np

import synth


def test_philox_known_answer():
    # Known-answer vectors of Philox4x32-10 published with the Random123 library
    # (counter, key) -> output.
    out = synth.philox4x32_10([0], [0], [0], [0], 0, 0)
    assert [int(o[0]) for o in out] == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]
    m = 0xFFFFFFFF
    out = synth.philox4x32_10([m], [m], [m], [m], m, m)
    assert [int(o[0]) for o in out] == [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]


def test_distribution_statistics():
    W = synth.student_t_host((512, 2048), seed=0, stream=0).astype(np.float64).ravel()
    base = W[np.abs(W) < 0.5]
    # std of the mixture: 0.02 * sqrt(0.999 + 0.001 * 400)
    assert abs(W.std() / (0.02 * np.sqrt(1.399)) - 1) < 0.08
    assert abs(W.mean()) < 2e-4
    assert abs(np.median(W)) < 2e-4
    # heavy tail: t(4) kurtosis is infinite; the sample excess kurtosis is large
    k = ((base - base.mean()) ** 4).mean() / base.var() ** 2 - 3
    assert k > 3
    # outlier fraction ~1e-3: fraction beyond 8 sd of the base distribution
    frac = np.mean(np.abs(W) > 0.02 * 8)
    assert 3e-4 < frac < 3e-3


def test_seed_and_stream_change_the_draws():
    a = synth.student_t_host((64, 64), seed=1, stream=0)
    b = synth.student_t_host((64, 64), seed=1, stream=1)
    c = synth.student_t_host((64, 64), seed=2, stream=0)
    d = synth.student_t_host((64, 64), seed=1, stream=0)
    assert np.array_equal(a.view(np.uint16), d.view(np.uint16))
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    # a slice is the same elements of the whole (counter = flat index)
    e = synth.student_t_host((10,), seed=1, stream=0, start=64 * 3)
    assert np.array_equal(e.view(np.uint16), a.reshape(-1)[64 * 3:64 * 3 + 10].view(np.uint16))


def test_shapes():
    s7 = synth.llama2_7b_shapes()
    assert sum(o * i for o, i in s7.values()) * 32 == 6_476_005_376
    s70 = synth.llama2_70b_shapes()
    assert sum(o * i for o, i in s70.values()) * 80 == 68_451_041_280
