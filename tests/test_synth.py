"""The seeded input generator: determinism, distribution, bf16 rounding."""
import numpy as np
import torch

import synth


def test_deterministic_and_offset_consistent():
    a = synth.bf16_bits((4096,), 3, "k")
    b = synth.bf16_bits((4096,), 3, "k")
    assert np.array_equal(a, b)
    part = np.empty(1000, dtype=np.uint16)
    synth.fill_bf16_into(part.ctypes.data, 1000, 3, "k", 1.0, offset=2000)
    assert np.array_equal(part, a[2000:3000])


def test_streams_differ_by_seed_and_tensor():
    a = synth.bf16_bits((2048,), 0, "q")
    assert not np.array_equal(a, synth.bf16_bits((2048,), 1, "q"))
    assert not np.array_equal(a, synth.bf16_bits((2048,), 0, "k"))


def test_standard_normal_moments():
    z = synth.normal_f64((1 << 20,), 0, "v")
    assert abs(z.mean()) < 5e-3
    assert abs(z.var() - 1.0) < 5e-3
    assert abs((z ** 4).mean() - 3.0) < 5e-2          # Gaussian kurtosis
    assert abs(np.mean(z < 0) - 0.5) < 2e-3


def test_factor_scales_values():
    z1 = synth.normal_f64((1000,), 5, "wq", 1.0)
    z2 = synth.normal_f64((1000,), 5, "wq", 0.02)
    np.testing.assert_allclose(z2, z1 * 0.02, rtol=1e-15)


def test_bf16_bits_are_rne_of_the_double_stream():
    z = synth.normal_f64((50000,), 9, "x", 0.5)
    bits = synth.bf16_bits((50000,), 9, "x", 0.5)
    # widen and check: the bf16 value is the nearest bf16 to z (ties even)
    w = synth.bf16_bits_to_f64(bits)
    exp = np.floor(np.log2(np.abs(z)))
    ulp = 2.0 ** (exp - 7)
    assert np.all(np.abs(w - z) <= ulp / 2 + 1e-300)
    # float32-representable inputs agree with torch's float32 -> bf16 (RNE)
    f = z.astype(np.float32).astype(np.float64)
    mine = np.array([synth.double_to_bf16_bits(x) for x in f[:3000]], dtype=np.uint16)
    ref = torch.from_numpy(f[:3000].astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_double_to_bf16_ties_and_specials():
    assert synth.double_to_bf16_bits(1.0 + 2 ** -8) == 0x3F80            # tie to even (down)
    assert synth.double_to_bf16_bits(1.0 + 3 * 2 ** -8) == 0x3F82        # tie to even (up)
    assert synth.double_to_bf16_bits(1.0 + 2 ** -8 + 2 ** -40) == 0x3F81  # above tie
    assert synth.double_to_bf16_bits(-2.0) == 0xC000
    assert synth.double_to_bf16_bits(0.0) == 0x0000
    assert synth.double_to_bf16_bits(1e300) == 0x7F80
    assert synth.double_to_bf16_bits(2.0 ** -130) == 0x0008               # subnormal grid 2^-133


def test_sample_rows_include_required_and_sorted():
    r = synth.sample_rows(1024, 200000, 0x5A17, must_include=[0, 199999, 127, 128])
    assert len(r) >= 1024 and np.all(np.diff(r) > 0)
    assert {0, 199999, 127, 128} <= set(r.tolist())
    assert r.min() >= 0 and r.max() < 200000
