"""The shared input generator: published SplitMix64 outputs, determinism,
thread-count independence and exact bf16 rounding."""
import numpy as np

import seeded_inputs


def test_splitmix64_published_sequence():
    # Vigna's splitmix64.c seeded with 1234567 emits these first two outputs.
    assert seeded_inputs.splitmix64_at(1234567, 0) == 6457827717110365317
    assert seeded_inputs.splitmix64_at(1234567, 1) == 3203168211198807973


def test_deterministic_and_thread_independent():
    a = seeded_inputs.normal_f32(7, (300001,), threads=1)
    b = seeded_inputs.normal_f32(7, (300001,), threads=7)
    assert np.array_equal(a, b)
    c = seeded_inputs.normal_f32(8, (300001,), threads=3)
    assert not np.array_equal(a, c)


def test_moments():
    a = seeded_inputs.normal_f32(9, (1 << 20,)).astype(np.float64)
    assert abs(a.mean()) < 5e-3
    assert abs(a.std() - 1.0) < 5e-3


def test_bf16_is_round_to_nearest_even_of_f32():
    f = seeded_inputs.normal_f32(10, (1 << 16,))
    b = seeded_inputs.normal_bf16_bits(10, (1 << 16,))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    expect = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    assert np.array_equal(b, expect)
    back = seeded_inputs.bf16_bits_to_f32(b)
    assert np.all(np.abs(back - f) <= np.abs(f) * 2.0 ** -8)
