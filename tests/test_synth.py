"""The seeded input generator (no GPU)."""
import numpy as np

import synth


def test_splitmix64_published_vector():
    # SplitMix64 from state 1234567: the first five outputs of the reference
    # generator (Steele, Lea, Flood 2014), as listed in common test suites.
    got = synth.splitmix64(1234567, 5).tolist()
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def test_normal_is_deterministic_and_standard():
    a = synth.normal(42, (200000,), np.float64)
    b = synth.normal(42, (200000,), np.float64)
    assert np.array_equal(a, b)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    assert not np.array_equal(a, synth.normal(43, (200000,), np.float64))


def test_fp16_rounding_is_nearest_even():
    z = synth.normal_f64(9, (5000,))
    h = synth.normal(9, (5000,), np.float16)
    assert np.array_equal(h, z.astype(np.float16))
    err = np.abs(h.astype(np.float64) - z)
    assert np.all(err <= np.abs(z) * 2.0 ** -11 + 2.0 ** -25)


def test_step_set_shapes():
    calls = synth.unet_step_set()
    assert len(calls) == 32
    assert sum(c.flops for c in calls) == 252_104_540_160   # 252.1 GFLOP per step
    assert {c.d for c in calls} == {40, 80, 160}
    assert sum(1 for c in calls if c.M == 77) == 16
    assert sum(1 for c in calls if c.N == 4096 and c.M == 4096) == 5


def test_seeds_distinct_per_tensor_and_call():
    s = set()
    for stream in range(1, 8):
        for call in range(32):
            s.update(synth.seeds(stream, call))
    assert len(s) == 7 * 32 * 3
