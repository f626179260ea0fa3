"""The seeded input generator (synthetic/), which feeds both the oracle and
the library: splitmix64 as published, bf16 rounding to nearest even, normals
with the moments of N(0, 1), and the decode lengths' range.  Parity cannot
catch a mistake here (both sides read the same inputs), so it is pinned on
its own."""
import numpy as np

import synthetic


def test_splitmix64_matches_the_published_sequence():
    # the first outputs of splitmix64 from state 0: the counter c yields the
    # output for state c * golden ratio constant (c = 0, 1, 2)
    golden = np.uint64(0x9E3779B97F4A7C15)
    with np.errstate(over="ignore"):
        ctr = np.arange(3, dtype=np.uint64) * golden
    got = [int(x) for x in synthetic.splitmix64(ctr)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_bf16_rounding_is_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20, -2.5, 0.0, -0.0,
                  np.inf, 3.0e38], np.float32)
    bits = synthetic.f32_to_bf16_bits(x)
    assert [int(b) for b in bits[:7]] == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC020, 0x0000, 0x8000]
    assert int(bits[7]) == 0x7F80
    back = synthetic.bf16_bits_to_f32(bits)
    assert np.isfinite(back[8]) and abs(float(back[8]) - 3.0e38) <= 3.0e38 * 2 ** -9  # large values stay finite
    assert np.array_equal(back[:7], np.array([1.0, 1.0, 1.0 + 2 ** -6, 1.0 + 2 ** -7, -2.5, 0.0, -0.0], np.float32))


def test_normals_have_the_moments_of_a_standard_normal():
    n = 1 << 20
    x = synthetic.normal(1234, synthetic.TID_Q, n, "f32").astype(np.float64)
    assert abs(x.mean()) < 5 / np.sqrt(n)
    assert abs(x.var() - 1.0) < 5 * np.sqrt(2.0 / n)
    assert abs((x ** 3).mean()) < 5 * np.sqrt(15.0 / n)          # skewness 0
    assert abs((x ** 4).mean() - 3.0) < 5 * np.sqrt(96.0 / n)   # kurtosis 3
    # about 4.55 % beyond two standard deviations
    assert abs((np.abs(x) > 2).mean() - 0.0455) < 0.002


def test_streams_are_independent_and_reproducible():
    a = synthetic.normal(7, synthetic.TID_K, 4096, "f32")
    assert np.array_equal(a, synthetic.normal(7, synthetic.TID_K, 4096, "f32"))
    b = synthetic.normal(7, synthetic.TID_V, 4096, "f32")
    c = synthetic.normal(8, synthetic.TID_K, 4096, "f32")
    for y in (b, c):
        assert abs(np.corrcoef(a, y)[0, 1]) < 5 / np.sqrt(4096)
    # an element range drawn on its own equals the same range of the whole stream
    assert np.array_equal(synthetic.normal(7, synthetic.TID_K, 1000, "f32", start=1000), a[1000:2000])


def test_decode_lengths_are_uniform_on_their_range():
    lens = synthetic.seqlens(2005, 20000)
    assert lens.min() >= 1024 and lens.max() <= 8192
    assert abs(lens.mean() - (1024 + 8192) / 2) < 5 * (8192 - 1024) / np.sqrt(12 * 20000)
    # a sample of the first sequences of a batch is the batch's first sequences
    lens64 = synthetic.seqlens(2005, 64)
    assert np.array_equal(lens64[:8], synthetic.seqlens(2005, 8))
    kc = synthetic.kv_cache(3, synthetic.TID_K, 4, 64, 2, 8, np.array([64, 10, 0, 33], np.int32))
    kc2 = synthetic.kv_cache(3, synthetic.TID_K, 2, 64, 2, 8, np.array([64, 10], np.int32))
    assert np.array_equal(kc[:2], kc2)
