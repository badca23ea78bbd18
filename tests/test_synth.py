"""The seeded input generator: determinism, independence of streams, the
distributions the workloads call for, and piecewise generation."""
import numpy as np

import synth


def test_deterministic_and_keyed():
    k = synth.key(0, synth.K_WQ, 3)
    a = synth.normal_bf16((1000,), k, 0.02)
    b = synth.normal_bf16((1000,), k, 0.02)
    np.testing.assert_array_equal(a, b)
    c = synth.normal_bf16((1000,), synth.key(0, synth.K_WQ, 4), 0.02)
    assert np.mean(a == c) < 0.05
    assert synth.key(0, 1, 2, 3) != synth.key(0, 1, 3, 2)


def test_piecewise_equals_whole():
    k = synth.key(7, 1)
    whole = synth.normal_bf16((1001,), k, 1.0)
    for first, n in [(0, 10), (1, 10), (3, 500), (999, 2), (500, 501)]:
        part = synth.normal_bf16((n,), k, 1.0, first=first)
        np.testing.assert_array_equal(part, whole[first:first + n])


def test_normal_moments():
    x = synth.normal_f32(400_000, synth.key(1, 2), 0.02).astype(np.float64)
    assert abs(x.mean()) < 0.02 * 0.01
    assert abs(x.std() - 0.02) < 0.02 * 0.01
    # bf16 rounding of the same stream stays within half an ulp (2^-9 relative)
    b = synth.bf16_bits_to_f32(synth.normal_bf16((400_000,), synth.key(1, 2), 0.02)).astype(np.float64)
    assert np.all(np.abs(b - x) <= np.abs(x) * 2.0 ** -8 + 1e-30)
    # standard-normal fraction beyond 2 sigma ~ 4.55 %
    assert abs(np.mean(np.abs(x) > 0.04) - 0.0455) < 0.002


def test_uniform_ints():
    t = synth.uniform_i32(200_000, synth.key(2), 0, 128256)
    assert t.min() >= 0 and t.max() < 128256
    assert abs(t.mean() - 128255 / 2) < 128256 * 0.005
    lengths = synth.uniform_i32(100_000, synth.key(3), 512, 4097)
    assert lengths.min() == 512 and lengths.max() == 4096


def test_workload_shapes():
    assert synth.LLAMA_1B.n_params() == 1_235_814_400
    assert synth.LLAMA_8B.n_params() == 8_030_261_248
    assert synth.TINY.n_params() == 3_015_936
    w = synth.WORKLOADS["llama1b_b16"]
    L = w.lengths()
    assert L.shape == (16,) and L.min() >= 512 and L.max() <= 4096
    np.testing.assert_array_equal(L, w.lengths())


def test_kv_prefix_fill():
    s = synth.TINY
    k, v = synth.alloc_kv(s, 2, 20)
    synth.fill_kv_prefix(s, k, v, [5, 9])
    assert np.all(k[:, 0, :, 5:] == 0) and np.any(k[:, 0, :, :5] != 0)
    assert np.all(v[:, 1, :, 9:] == 0) and np.any(v[:, 1, :, :9] != 0)
    assert not np.array_equal(k[:, 1, :, :5], v[:, 1, :, :5])
