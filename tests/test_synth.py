"""The seeded input generator: determinism, distribution, bf16 rounding and the
8-bit (E4M3) input recipe."""

import numpy as np
import pytest

import oracle
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


def test_e4m3_quantised_inputs_follow_the_recipe():
    """The 8-bit input recipe: per 128-row tile, scale = the tile's largest
    magnitude / 448 (its largest element becomes +-448 exactly) and every code
    is within half an E4M3 step of x / scale (relative 2^-4 for normal values,
    absolute 2^-10 in the subnormal range)."""
    import torch

    x = synth.bf16_bits_to_f64(synth.normal_bf16(951, (2, 3, 300, 64)))
    codes, scales = synth.normal_e4m3(951, (2, 3, 300, 64))
    assert codes.dtype == np.uint8 and scales.shape == (2, 3, 3)
    deq = oracle.e4m3_to_f64(codes)
    for t in range(3):
        rows = slice(128 * t, min(128 * (t + 1), 300))
        xt = x[:, :, rows]
        amax = np.max(np.abs(xt), axis=(2, 3))
        assert np.allclose(scales[:, :, t], (amax / 448.0).astype(np.float32), rtol=1e-7)
        assert np.max(np.abs(deq[:, :, rows]), axis=(2, 3)).tolist() == [[448.0] * 3] * 2
        y = xt / scales[:, :, t][..., None, None].astype(np.float64)
        err = np.abs(deq[:, :, rows] - y)
        bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6)
        assert np.all(err <= bound)
    # the device twin quantises the same values the same way
    c2, s2 = synth.quantize_e4m3_tiles(torch.from_numpy(x.astype(np.float32)))
    assert np.array_equal(c2.numpy(), codes) and np.array_equal(s2.numpy(), scales)


def test_block_draws_equal_the_full_tensor_slice():
    """A head drawn at its own counters equals that head of the full tensor."""
    full = synth.normal_bf16(4321, (2, 3, 5, 8))
    for b in range(2):
        for h in range(3):
            assert np.array_equal(synth.normal_bf16_block(4321, (2, 3, 5, 8), (b, h)), full[b, h])
    assert np.array_equal(synth.normal_bf16_block(4321, (2, 3, 5, 8), (1,)), full[1])
    assert np.array_equal(synth.normal_bf16_block(4321, (2, 3, 5, 8), (1, 2, 4)), full[1, 2, 4])
    assert np.array_equal(synth.normal_bf16_block(4321, (2, 3, 5, 8), (1, 1), first=3),
                          full[1, 1, :3])
    with pytest.raises(IndexError):
        synth.normal_bf16_block(4321, (2, 3, 5, 8), (2, 0))
