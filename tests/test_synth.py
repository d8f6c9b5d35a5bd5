"""The seeded input generator: published SplitMix64 values, bf16 rounding, slicing."""
import numpy as np

import synth


def test_splitmix64_published_seed0_sequence():
    # first outputs of SplitMix64 from state 0 (Steele, Lea, Flood 2014 reference generator)
    got = [int(v) for v in synth.splitmix64(0, 0, 3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20, -2.5, 0.0],
                 np.float32)
    assert synth.f32_to_bf16_bits(x).tolist() == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC020, 0x0000]
    assert synth.bf16_bits_to_f64(np.array([0x3F81], np.uint16))[0] == 1.0 + 2 ** -7


def test_normal_moments_and_slices():
    x = synth.normal(3, 1 << 20)
    assert abs(x.mean()) < 5e-3 and abs(x.var() - 1) < 5e-3
    assert np.array_equal(synth.normal(3, 1001, start=777), x[777:1778])
    a = synth.qkv_bf16(2, 10, 3, 8, "k")
    b = synth.qkv_bf16(2, 4, 3, 8, "k", token_offset=6)
    assert np.array_equal(a[6:], b)
    assert not np.array_equal(synth.qkv_bf16(2, 10, 3, 8, "q"), a)
