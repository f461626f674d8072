"""The seeded input generator: determinism, distribution and bf16 rounding."""

import numpy as np

import synth


def test_deterministic_and_distinct_streams():
    a = synth.normal_bf16(7, (4, 1000))
    b = synth.normal_bf16(7, (4, 1000))
    c = synth.normal_bf16(8, (4, 1000))
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)


def test_standard_normal_moments():
    x = synth.bf16_bits_to_f64(synth.normal_bf16(3, (200000,)))
    assert abs(x.mean()) < 0.01
    assert abs(x.var() - 1.0) < 0.01
    # tail mass beyond 3 sigma close to 0.27 %
    assert 0.0015 < np.mean(np.abs(x) > 3) < 0.0040


def test_bf16_round_to_nearest_even():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0])
    got = synth.bf16_bits_to_f64(synth.f64_to_bf16_bits(x))
    assert list(got) == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 0.0]
    # widening is exact and round-trips
    bits = synth.normal_bf16(5, (1000,))
    assert np.array_equal(synth.f64_to_bf16_bits(synth.bf16_bits_to_f64(bits)), bits)


def test_uniform_int_range():
    k = synth.uniform_int(9, 10000, 1024, 32768)
    assert k.min() >= 1024 and k.max() <= 32768
    assert abs(k.mean() - (1024 + 32768) / 2) < 400
