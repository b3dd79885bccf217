"""The seeded input generator: determinism, independence of streams, recipe shapes."""
import numpy as np

import synth


def _splitmix64_stream(origin, n):
    """splitmix64 from its published definition: state += golden; output = mix(state)."""
    M = (1 << 64) - 1
    out, state = [], origin
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & M
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
        out.append(z ^ (z >> 31))
    return out


def test_counter_draws_follow_splitmix64():
    # the stream origin is itself one splitmix64 mix of (seed, tensor id)
    M = (1 << 64) - 1
    seed, tid = 0, 5
    pre = (seed * 0x9E3779B97F4A7C15 + tid * 0xD1B54A32D192ED03 + 0x2545F4914F6CDD1D) & M
    z = pre
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
    origin = z ^ (z >> 31)
    assert list(synth.raw_u64(seed, tid, 16)) == _splitmix64_stream(origin, 16)


def test_deterministic_and_streams_differ():
    a = synth.normal_f32(0, 1, (1000,))
    b = synth.normal_f32(0, 1, (1000,))
    c = synth.normal_f32(0, 2, (1000,))
    assert np.array_equal(a, b) and not np.array_equal(a, c)


def test_normal_statistics():
    x = synth.normal_f64(3, 7, (400000,))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01


def test_activation_recipe():
    xb, chans = synth.activation_bf16(0, 64, 256, 0.02, 20.0)
    assert xb.shape == (64, 256) and xb.dtype == np.uint16
    assert len(chans) == 5 and len(set(chans.tolist())) == 5
    x = synth.bf16_bits_to_f32(xb)
    col_std = x.std(axis=0)
    assert np.all(col_std[chans] > 8) and np.median(col_std) < 1.5


def test_outlier_counts_of_workloads():
    assert synth.outlier_count(0.01, 3072) == 31
    assert synth.outlier_count(0.01, 12288) == 123
    assert synth.outlier_count(0.005, 4096) == 20
    assert synth.outlier_count(0.005, 14336) == 72
    assert synth.outlier_count(0.02, 256) == 5
