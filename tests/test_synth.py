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


def test_norm_weights_unit_or_seeded():
    s = synth.TINY
    ones = synth.bf16_bits_to_f32(synth.make_norm(s, synth.K_ATTN_NORM, 0))
    assert np.all(ones == 1.0)
    g0 = synth.bf16_bits_to_f32(synth.make_norm(s, synth.K_ATTN_NORM, 0, 0.3)).astype(np.float64)
    g1 = synth.bf16_bits_to_f32(synth.make_norm(s, synth.K_ATTN_NORM, 1, 0.3)).astype(np.float64)
    gf = synth.bf16_bits_to_f32(synth.make_norm(s, synth.K_FFN_NORM, 0, 0.3)).astype(np.float64)
    # distinct vectors per norm and layer, around 1 with the asked spread
    assert not np.array_equal(g0, g1) and not np.array_equal(g0, gf)
    big = synth.bf16_bits_to_f32(synth.normal_bf16_mean((200_000,), synth.key(0, synth.K_FFN_NORM, 3), 1.0, 0.3))
    assert abs(big.astype(np.float64).mean() - 1.0) < 0.005 and abs(big.astype(np.float64).std() - 0.3) < 0.005
    # the offset stream is the plain stream plus the mean, rounded once
    k = synth.key(5, 9)
    plain = synth.normal_f32(1000, k, 0.3)
    shifted = synth.bf16_bits_to_f32(synth.normal_bf16_mean((1000,), k, 1.0, 0.3)).astype(np.float64)
    ref = (np.float32(1.0) + plain).astype(np.float64)
    assert np.all(np.abs(shifted - ref) <= np.abs(ref) * 2.0 ** -8)
    m = synth.make_model(s, norm_sigma=0.3)
    m1 = synth.with_norms(synth.make_model(s), s, 0.3)
    for name in ("attn_norm", "ffn_norm"):
        np.testing.assert_array_equal(m["layers"][1][name], m1["layers"][1][name])
    np.testing.assert_array_equal(m["final_norm"], m1["final_norm"])
    assert np.any(synth.bf16_bits_to_f32(m["final_norm"]) != 1.0)
