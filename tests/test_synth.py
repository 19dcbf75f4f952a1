"""The seeded input generator: published SplitMix64 outputs, Box-Muller, bf16 rounding."""
import math

import numpy as np

import synth


def test_splitmix64_published_outputs():
    """First outputs of SplitMix64 seeded with 1234567 (published reference sequence)."""
    expect = [6457827717110365317, 3203168211198807973, 9817491932198370423,
              4593380528125082431, 16408922859458223821]
    assert [synth.splitmix64_at(1234567, n) for n in range(5)] == expect


def _py_normal(seed, tid, i):
    M = (1 << 64) - 1

    def sm(s, n):
        z = (s + (n + 1) * 0x9E3779B97F4A7C15) & M
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
        return z ^ (z >> 31)
    key = sm(seed, tid)
    u1 = 1.0 - (sm(key, 2 * i) >> 11) * 2.0 ** -53
    u2 = (sm(key, 2 * i + 1) >> 11) * 2.0 ** -53
    return math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2)


def test_normal_matches_python_definition_and_offsets():
    got = synth.normal((40,), 7, seed=3)
    ref = [_py_normal(3, 7, i) for i in range(40)]
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)
    tail = synth.normal((10,), 7, seed=3, first=30)
    np.testing.assert_array_equal(tail, got[30:])


def test_normal_moments():
    x = synth.normal((1 << 20,), 2, mean=0.5, std=math.sqrt(2.0))
    assert abs(x.mean() - 0.5) < 5 * math.sqrt(2.0 / x.size)
    assert abs(x.var() - 2.0) < 0.02


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.140625],
                    np.float32)
    bits = synth.f32_to_bf16(vals)
    back = synth.bf16_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to the even mantissa (1.0).
    np.testing.assert_array_equal(back, [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5, 3.140625])


def test_bf16_stream_is_rounded_f32_stream():
    a = synth.normal((1000,), 4, dtype="bf16")
    f = synth.normal((1000,), 4, dtype="f32")
    np.testing.assert_array_equal(a, synth.f32_to_bf16(f))


def test_workload_table():
    w = synth.BY_NAME["bf16_F1024_P2560_C320"]
    assert (w.F, w.N, w.L, w.P, w.C, w.heads * w.d) == (1024, 64, 16, 2560, 320, 320)
    assert w.tokens == 1024 * 2560
    for w in synth.WORKLOADS:
        assert w.F % w.N == 0 and w.heads * w.d == w.C and w.C % w.groups == 0
