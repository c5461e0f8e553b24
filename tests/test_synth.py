"""The seeded input generator (CPU): determinism, counter addressing, distributions."""
import math

import numpy as np

import synth
from synth import workloads


def test_known_splitmix_outputs():
    """Counter mode reproduces the published SplitMix64 stream: with seed state s, output i is
    mix64(s + (i+1)*GAMMA).  Reference values of the sequential generator seeded with 0
    (Vigna's splitmix64.c): 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F."""
    expect = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    mix = lambda z: _mix64(z)
    got = [mix((i + 1) * 0x9E3779B97F4A7C15 % (1 << 64)) for i in range(3)]
    assert got == expect


def _mix64(z):
    M = (1 << 64) - 1
    z &= M
    z ^= z >> 30
    z = (z * 0xBF58476D1CE4E5B9) & M
    z ^= z >> 27
    z = (z * 0x94D049BB133111EB) & M
    z ^= z >> 31
    return z


def test_counter_stream_matches_python_model():
    seed, tensor, seq = 123, synth.Q, 7
    G = 0x9E3779B97F4A7C15
    M = (1 << 64) - 1
    k = _mix64(seed + G)
    k = _mix64(k + (tensor + 1) * G)
    k = _mix64(k + (seq + 1) * G)
    ref = [_mix64(k + (i + 1) * G) for i in range(100, 110)]
    assert synth.raw_bits(seed, tensor, seq, 100, 10).tolist() == ref


def test_sub_blocks_are_slices_of_the_whole():
    full = synth.bf16_normal(5, synth.X, 3, 64, 0, 40)
    blk = synth.bf16_normal(5, synth.X, 3, 64, 10, 25, 8, 40)
    np.testing.assert_array_equal(full[10:25, 8:40], blk)


def test_streams_differ_and_repeat():
    a = synth.bf16_normal(1, synth.X, 0, 32, 0, 8)
    b = synth.bf16_normal(1, synth.X, 1, 32, 0, 8)
    c = synth.bf16_normal(1, synth.A, 0, 32, 0, 8)
    assert (a != b).mean() > 0.9 and (a != c).mean() > 0.9
    np.testing.assert_array_equal(a, synth.bf16_normal(1, synth.X, 0, 32, 0, 8))


def test_distributions():
    z = synth.bf16_to_f64(synth.bf16_normal(9, synth.X, 0, 1000, 0, 400))
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    assert abs(np.mean(np.abs(z) > 1.96) - 0.05) < 0.003
    u = synth.f32_uniform(9, synth.W, 0, 1000, 0, 100)
    assert u.min() >= 0 and u.max() < 1 and abs(u.mean() - 0.5) < 0.01
    b = synth.f32_normal(9, synth.BIAS_C, 0, 1000, 0, 100, scale=0.5)
    assert abs(b.std() - 0.5) < 0.01


def test_generator_log_cos_accuracy():
    lib = synth.host_lib()
    rng = np.random.default_rng(0)
    for u in rng.random(2000):
        u = float(u) or 1.0
        assert abs(lib.synth_log_host(u) - math.log(u)) <= 4e-16 * max(1.0, abs(math.log(u)))
    for t in rng.random(2000):
        assert abs(lib.synth_cos2pi_host(float(t)) - math.cos(2 * math.pi * float(t))) < 1e-15


def test_ragged_lengths_in_range():
    wl = workloads.ragged_decode()
    assert wl.B == 32 and all(32768 <= n <= 131072 for n in wl.n0)
    assert len(set(wl.n0)) > 25
