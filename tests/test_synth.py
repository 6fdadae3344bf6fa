"""The seeded input generator: published splitmix64 values, determinism, distributions."""
import numpy as np

import synth


def test_splitmix64_published_values():
    # First three outputs of splitmix64 from state 0 (Vigna's reference generator).
    z = synth.splitmix64(0, 3)
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_based_offsets():
    full = synth.splitmix64(1234, 10)
    assert np.array_equal(synth.splitmix64(1234, 4, start=6), full[6:])


def test_uniform_range_and_normal_moments():
    u = synth.uniform01(7, 100000)
    assert u.min() > 0.0 and u.max() <= 1.0
    x = synth.normal(8, 200000, std=0.02)
    assert abs(x.std() - 0.02) < 0.0005 and abs(x.mean()) < 0.0005


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 is halfway between bf16 1.0 and 1 + 2^-7: ties go to even (1.0).
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9, -2.5], dtype=np.float32)
    assert [hex(int(b)) for b in synth.f32_to_bf16_bits(x)] == ["0x3f80", "0x3f82", "0x3f80", "0xc020"]


def test_workloads_deterministic_and_shaped():
    a1, w1 = synth.router(4)
    a2, w2 = synth.router(16)
    assert np.array_equal(a1, a2[:4]) and np.array_equal(w1, w2)
    assert a2.shape == (16, 2560) and w2.shape == (512, 2560)
    a, w = synth.narrow(512, w_index=3)
    assert w.shape == (96, 2560) and a.dtype == np.uint16
    _, w0 = synth.narrow(512, w_index=0)
    assert not np.array_equal(w, w0)
    _, wa = synth.chunk(150, 512)
    _, wb = synth.chunk(150, 640)
    assert np.array_equal(wa, wb[:512])


def test_integer_bits_exact():
    for fmt in ("bf16", "f16"):
        b = synth.integer_bits(3, (1000,), fmt, -15, 15)
        v = synth.bits_to_float32(b, fmt)
        assert np.array_equal(v, np.round(v)) and v.min() >= -15 and v.max() <= 15
