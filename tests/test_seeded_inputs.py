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


def test_e4m3_rounding_matches_torch_cast():
    """The generator's E4M3 rounding (nearest even) equals torch's float32 ->
    float8_e4m3fn cast on N(0, 1) samples, on every representable value, on
    the midpoints between neighbours (ties go to the even mantissa) and on the
    subnormal range; values beyond 448 saturate to +-448."""
    import torch
    f = seeded_inputs.normal_f32(11, (200000,), scale=3.0)
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(seeded_inputs.normal_e4m3_bits(11, (200000,), scale=3.0), ref)
    codes = np.arange(256, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    fin = np.isfinite(vals)
    pos = np.unique(vals[fin & (vals >= 0)])
    mids = ((pos[1:].astype(np.float64) + pos[:-1]) / 2).astype(np.float32)
    probes = np.concatenate([vals[fin], mids, -mids, np.linspace(0, 2 ** -6, 97, dtype=np.float32)])
    ref = torch.from_numpy(probes).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(seeded_inputs.round_e4m3_bits(probes), ref)
    sat = seeded_inputs.round_e4m3_bits(np.array([448.0, 470.0, 1e6, -1e6], dtype=np.float32))
    assert list(sat) == [0x7E, 0x7E, 0x7E, 0xFE]
