"""Pins of the CPU oracle to things other than itself.

The pages print no worked numeric example (they only name the fused
operations: "Hazy megakernel summary" page, section 四(二)), so each pin here
is a closed form, an invariant, a special case that reduces to a library
routine (numpy), or brute force on tiny inputs.  Each is chosen so that a
plausible slip in the oracle (a dropped eps or gamma, a wrong RoPE pairing,
sign or frequency, a missing 1/sqrt(d), a wrong GQA group, swapped SwiGLU
operands, a mis-wired residual or norm weight, an off-by-one position) fails
at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
import synth

PRECS = ["f64", "f32"]
U = {"f64": 2.0 ** -53, "f32": 2.0 ** -24}


def bf16(x: float) -> int:
    """bf16 bit pattern of a value that is exactly representable in bf16."""
    u = np.array([x], dtype=np.float32).view(np.uint32)[0]
    assert (u & 0xFFFF) == 0, x
    return int(u >> 16)


def widen(bits) -> np.ndarray:
    return synth.bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


def bf16_grid_neighbours(x: float):
    """All bf16 values within 2 ulp of x, by enumeration (brute force)."""
    f = np.float32(x)
    u = int(np.array([f], dtype=np.float32).view(np.uint32)[0]) >> 16
    cands = [(u + k) & 0xFFFF for k in range(-3, 4)]
    return cands


# ----------------------------------------------------------------------------- bf16

@pytest.mark.parametrize("prec", PRECS)
def test_bf16_widening_exact(prec):
    for bits, val in [(0x3F80, 1.0), (0xC000, -2.0), (0x3F81, 1.0078125), (0x0000, 0.0),
                      (0x4B80, 16777216.0), (0x3C23, 0.0099487304688)]:
        got = oracle.bf16_to_real(bits, prec)
        assert got == pytest.approx(val, rel=0, abs=1e-12) if bits != 0x3C23 else abs(got - val) < 1e-9


@pytest.mark.parametrize("prec", PRECS)
def test_bf16_round_nearest_even_ties(prec):
    # 1 + 2^-8 lies halfway between 1.0 (even) and 1.0078125 (odd): goes to 1.0
    assert oracle.real_to_bf16(1.0 + 2.0 ** -8, prec) == 0x3F80
    # 1 + 3*2^-8 lies halfway between 0x3F81 (odd) and 0x3F82 (even): goes up
    assert oracle.real_to_bf16(1.0 + 3 * 2.0 ** -8, prec) == 0x3F82
    assert oracle.real_to_bf16(-(1.0 + 2.0 ** -8), prec) == 0xBF80
    assert oracle.real_to_bf16(0.0, prec) == 0x0000


@pytest.mark.parametrize("prec", PRECS)
def test_bf16_round_is_nearest_by_enumeration(prec):
    rng = np.random.default_rng(5)
    xs = np.concatenate([rng.normal(0, 1, 400), rng.normal(0, 0.02, 400), rng.normal(0, 300, 200)])
    for x in xs:
        if prec == "f32":
            x = float(np.float32(x))
        got = oracle.real_to_bf16(float(x), prec)
        cands = bf16_grid_neighbours(x)
        dists = [abs(widen([c])[0] - x) for c in cands]
        best = min(dists)
        assert abs(widen([got])[0] - x) == best
        winners = [c for c, dd in zip(cands, dists) if dd == best]
        if len(winners) == 2:  # a tie: the even mantissa wins
            assert got % 2 == 0


# ----------------------------------------------------------------------------- RMSNorm

@pytest.mark.parametrize("prec", PRECS)
@pytest.mark.parametrize("c", [0.37, -2.5, 1e-3, 40.0])
def test_rmsnorm_constant_vector_closed_form(prec, c):
    n, eps = 256, 1e-5
    ones = np.full(n, bf16(1.0), dtype=np.uint16)
    y = oracle.rmsnorm(np.full(n, c), ones, eps, prec)
    want = math.copysign(1.0, c) / math.sqrt(1.0 + eps / (c * c))
    np.testing.assert_allclose(y, want, rtol=8 * U[prec] * 64, atol=0)


@pytest.mark.parametrize("prec", PRECS)
def test_rmsnorm_gamma_and_unit_mean_square(prec):
    rng = np.random.default_rng(1)
    n = 512
    x = rng.normal(0, 3, n)
    gvals = np.array([0.5, 2.0, -1.0, 0.25], dtype=np.float32)
    gamma = np.array([bf16(float(gvals[i % 4])) for i in range(n)], dtype=np.uint16)
    ones = np.full(n, bf16(1.0), dtype=np.uint16)
    y1 = oracle.rmsnorm(x, ones, 0.0, prec)
    # eps = 0: output has mean square exactly 1 and is invariant to positive scaling
    assert np.mean(y1.astype(np.float64) ** 2) == pytest.approx(1.0, rel=200 * U[prec] * n)
    y2 = oracle.rmsnorm(7.0 * x, ones, 0.0, prec)
    np.testing.assert_allclose(y2, y1, rtol=100 * U[prec] * n)
    # gamma multiplies elementwise
    yg = oracle.rmsnorm(x, gamma, 0.0, prec)
    np.testing.assert_allclose(yg, y1 * gvals[np.arange(n) % 4], rtol=8 * U[prec], atol=0)
    # eps enters under the root: a zero vector stays zero, a tiny one is damped
    z = oracle.rmsnorm(np.full(n, 1e-4), ones, 1e-5, prec)
    want = 1e-4 / math.sqrt(1e-8 + 1e-5)
    np.testing.assert_allclose(z, want, rtol=50 * U[prec] * 64)


# ----------------------------------------------------------------------------- RoPE

@pytest.mark.parametrize("prec", PRECS)
def test_rope_identity_at_position_zero(prec):
    v = np.random.default_rng(2).normal(size=64)
    if prec == "f32":
        v = v.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(oracle.rope(v, 0, 1e4, prec), v)


@pytest.mark.parametrize("prec", PRECS)
def test_rope_unit_pair_closed_form(prec):
    # d = 2: one pair, frequency theta^0 = 1, so (1, 0) turns to (cos p, sin p)
    for p in (1, 2, 7, 1000):
        r = oracle.rope(np.array([1.0, 0.0]), p, 1e4, prec)
        tol = 4 * U[prec] * max(1, p)
        assert r[0] == pytest.approx(math.cos(p), abs=tol)
        assert r[1] == pytest.approx(math.sin(p), abs=tol)


@pytest.mark.parametrize("prec", PRECS)
@pytest.mark.parametrize("theta", [1e4, 5e5])
def test_rope_pairs_norm_and_angle(prec, theta):
    d, p = 64, 37
    rng = np.random.default_rng(3)
    v = rng.normal(size=d)
    r = oracle.rope(v, p, theta, prec)
    h = d // 2
    for i in range(h):
        a0 = math.atan2(v[i + h], v[i])
        a1 = math.atan2(r[i + h], r[i])
        want = p * theta ** (-2.0 * i / d)
        diff = (a1 - a0 - want + math.pi) % (2 * math.pi) - math.pi
        assert abs(diff) < 1e-5 if prec == "f32" else abs(diff) < 1e-12
        assert math.hypot(r[i], r[i + h]) == pytest.approx(math.hypot(v[i], v[i + h]), rel=10 * U[prec])


@pytest.mark.parametrize("prec", PRECS)
def test_rope_couples_i_with_i_plus_half(prec):
    d = 16
    for i in range(d):
        e = np.zeros(d)
        e[i] = 1.0
        r = oracle.rope(e, 5, 1e4, prec)
        partner = (i + d // 2) % d
        nz = set(np.nonzero(np.abs(r) > 1e-12)[0].tolist())
        assert nz <= {i, partner}


# ----------------------------------------------------------------------------- attention

def _rand_bf16(shape, seed, sigma=1.0):
    return synth.normal_bf16(shape, synth.key(99, seed), sigma)


@pytest.mark.parametrize("prec", PRECS)
def test_attention_single_key_returns_v(prec):
    d = 64
    K, V = _rand_bf16((1, d), 1), _rand_bf16((1, d), 2)
    q = np.random.default_rng(4).normal(size=d)
    o = oracle.attention_head(q, K, V, prec)
    np.testing.assert_array_equal(o, widen(V[0]))


@pytest.mark.parametrize("prec", PRECS)
def test_attention_identical_keys_give_mean_of_v(prec):
    d, n = 64, 37
    K = np.repeat(_rand_bf16((1, d), 3), n, axis=0)
    V = _rand_bf16((n, d), 4)
    q = np.random.default_rng(5).normal(size=d)
    o = oracle.attention_head(q, K, V, prec)
    np.testing.assert_allclose(o, widen(V).mean(axis=0), rtol=0, atol=40 * U[prec] * n)


@pytest.mark.parametrize("prec", PRECS)
def test_attention_weights_closed_form_and_sum_to_one(prec):
    # V = identity rows expose the softmax weights; K_j = c_j e_0 and q = e_0 give
    # scores c_j / sqrt(d), so w_j = exp(c_j/sqrt d) / sum exp(c/sqrt d).
    d = 16
    cs = [1.0, -2.0, 0.5, 3.0, 0.0, 1.5]
    n = len(cs)
    K = np.zeros((n, d), dtype=np.uint16)
    for j, c in enumerate(cs):
        K[j, 0] = bf16(c)
    V = np.zeros((n, d), dtype=np.uint16)
    for j in range(n):
        V[j, j] = bf16(1.0)
    q = np.zeros(d)
    q[0] = 1.0
    o = oracle.attention_head(q, K, V, prec)
    e = [math.exp(c / math.sqrt(d)) for c in cs]
    want = [x / sum(e) for x in e]
    np.testing.assert_allclose(o[:n], want, rtol=20 * U[prec])
    assert np.all(o[n:] == 0)
    assert o.sum() == pytest.approx(1.0, abs=1e-6 if prec == "f32" else 1e-14)


@pytest.mark.parametrize("prec", PRECS)
def test_attention_large_scores_stay_finite(prec):
    d = 8
    K = np.zeros((3, d), dtype=np.uint16)
    K[:, 0] = [bf16(2816.0), bf16(2800.0), bf16(-2816.0)]
    V = np.zeros((3, d), dtype=np.uint16)
    V[:, 1] = [bf16(1.0), bf16(2.0), bf16(3.0)]
    q = np.zeros(d)
    q[0] = 1.0
    o = oracle.attention_head(q, K, V, prec)
    s = np.array([2816.0, 2800.0, -2816.0]) / math.sqrt(d)
    w = np.exp(s - s.max())
    w /= w.sum()
    assert np.isfinite(o).all()
    assert o[1] == pytest.approx(w[0] * 1 + w[1] * 2 + w[2] * 3, rel=1e-6)


# ----------------------------------------------------------------------------- silu / argmax

@pytest.mark.parametrize("prec", PRECS)
def test_silu_closed_forms(prec):
    assert oracle.silu(0.0, prec) == 0.0
    assert oracle.silu(1.0, prec) == pytest.approx(1 / (1 + math.exp(-1)), rel=4 * U[prec])
    assert oracle.silu(-1.0, prec) == pytest.approx(-1 / (1 + math.e), rel=4 * U[prec])
    assert oracle.silu(40.0, prec) == pytest.approx(40.0, rel=1e-15 if prec == "f64" else 1e-7)
    assert abs(oracle.silu(-40.0, prec)) < 1e-15


def test_argmax_first_maximum():
    rng = np.random.default_rng(6)
    for _ in range(50):
        x = rng.integers(-5, 5, size=97).astype(np.float64)  # many ties
        assert oracle.argmax(x) == int(np.argmax(x))  # numpy returns the first occurrence
        assert x[oracle.argmax(x)] == x.max()
    assert oracle.argmax(np.array([1.0, 3.0, 3.0])) == 1


# ----------------------------------------------------------------------------- matvec

def test_matvec_f64_matches_library_within_bound():
    rng = np.random.default_rng(7)
    W = synth.normal_bf16((300, 777), synth.key(98, 1), 0.02)
    x = rng.normal(size=777)
    y = oracle.matvec(W, x, "f64")
    Wf = widen(W)
    ref = Wf @ x
    bound = 777 * U["f64"] * (np.abs(Wf) @ np.abs(x)) * 2
    assert np.all(np.abs(y - ref) <= bound)


def test_matvec_f32_within_sequential_error_bound():
    rng = np.random.default_rng(8)
    n = 2048
    W = synth.normal_bf16((64, n), synth.key(98, 2), 0.02)
    x = rng.normal(size=n).astype(np.float32)
    y32 = oracle.matvec(W, x, "f32").astype(np.float64)
    Wf = widen(W)
    exact = Wf @ x.astype(np.float64)
    g = n * U["f32"] / (1 - n * U["f32"])
    assert np.all(np.abs(y32 - exact) <= g * (np.abs(Wf) @ np.abs(x.astype(np.float64))))


# ----------------------------------------------------------------------------- whole-step pins

def _tiny_kv(batch=1, max_seq=96):
    return synth.alloc_kv(synth.TINY, batch, max_seq)


@pytest.mark.parametrize("prec", PRECS)
def test_incremental_decode_equals_full_recompute(tiny_model, prec):
    s = synth.TINY
    orc = oracle.Oracle(s, tiny_model, prec)
    toks = synth.uniform_i32(12, synth.key(97, 1), 0, s.vocab)
    k1, v1 = _tiny_kv()
    full = orc.prefill(k1, v1, 0, toks, all_logits=True)
    k2, v2 = _tiny_kv()
    for p, t in enumerate(toks):
        lg = orc.decode_step(k2, v2, 0, int(t), p)
        # same operations in the same order: bitwise equal
        np.testing.assert_array_equal(lg, full[p])
    np.testing.assert_array_equal(k1, k2)
    np.testing.assert_array_equal(v1, v2)


def test_prefill_then_decode_equals_longer_prefill(tiny_model):
    s = synth.TINY
    orc = oracle.Oracle(s, tiny_model, "f64")
    toks = synth.uniform_i32(20, synth.key(97, 2), 0, s.vocab)
    k1, v1 = _tiny_kv()
    last = orc.prefill(k1, v1, 0, toks)
    k2, v2 = _tiny_kv()
    orc.prefill(k2, v2, 0, toks[:-1])
    lg = orc.decode_step(k2, v2, 0, int(toks[-1]), len(toks) - 1)
    np.testing.assert_array_equal(lg, last)


def test_f32_oracle_close_to_f64(tiny_model):
    s = synth.TINY
    toks = synth.uniform_i32(8, synth.key(97, 3), 0, s.vocab)
    outs = {}
    for prec in PRECS:
        k, v = _tiny_kv()
        outs[prec] = oracle.Oracle(s, tiny_model, prec).prefill(k, v, 0, toks)
    np.testing.assert_allclose(outs["f32"], outs["f64"], atol=1e-3, rtol=1e-3)


def _np_rms(x, g, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * g


def _silu(z):
    return z / (1 + np.exp(-z))


def test_position_zero_step_reduces_to_dense_algebra():
    """At position 0 attention sees one key, so it returns that key's V row;
    the rest of the step is then matrix-vector products (numpy) and the
    residual/norm wiring.  Distinct norm weights per site catch a swapped
    gamma, and an untied head catches a tied/untied mix-up."""
    s = synth.ModelShape(2, 128, 4, 2, 32, 256, 300, 1e-5, 1e4, False)
    m = synth.make_model(s)
    m["final_norm"] = np.full(s.hidden, bf16(0.5), dtype=np.uint16)
    for i, L in enumerate(m["layers"]):
        L["attn_norm"] = np.full(s.hidden, bf16(2.0 + i), dtype=np.uint16)
        L["ffn_norm"] = np.full(s.hidden, bf16(0.25 * (i + 1)), dtype=np.uint16)
    orc = oracle.Oracle(s, m, "f64")
    k, v = synth.alloc_kv(s, 1, 4)
    tok = 123
    logits, dump = orc.decode_step(k, v, 0, tok, 0, dump=True)
    grp = s.n_q_heads // s.n_kv_heads
    x = widen(m["embed"][tok])
    for l, L in enumerate(m["layers"]):
        W = {n: widen(L[n]) for n in synth.LAYER_TENSORS}
        a = _np_rms(x, W["attn_norm"], s.rms_eps)
        vv = W["wv"] @ a
        np.testing.assert_allclose(dump["v"][l], vv, rtol=1e-12, atol=1e-15)
        vrow = widen(v[l, 0].reshape(s.n_kv_heads, -1, s.head_dim)[:, 0, :])  # cache row 0
        o = np.concatenate([vrow[h // grp] for h in range(s.n_q_heads)])
        np.testing.assert_array_equal(dump["attn"][l], o)
        x = x + W["wo"] @ o
        np.testing.assert_allclose(dump["x_attn"][l], x, rtol=1e-12, atol=1e-14)
        b = _np_rms(x, W["ffn_norm"], s.rms_eps)
        act = _silu(W["w_gate"] @ b) * (W["w_up"] @ b)
        np.testing.assert_allclose(dump["act"][l], act, rtol=1e-10, atol=1e-15)
        x = x + W["w_down"] @ act
        np.testing.assert_allclose(dump["x_out"][l], x, rtol=1e-12, atol=1e-14)
    f = _np_rms(x, widen(m["final_norm"]), s.rms_eps)
    np.testing.assert_allclose(logits, widen(m["lm_head"]) @ f, rtol=1e-11, atol=1e-13)


def test_step_rotates_q_and_k_by_the_position_and_leaves_v():
    """At a position p > 0, the dumped q, k, v of layer 0 against the plain
    products W a (numpy, a = rms(embed row) * gamma): v is the product itself
    (not rotated); every (i, i + d/2) pair of q and k keeps its length and is
    turned by exactly p * theta^(-2i/d); the cache row written at p holds the
    bf16 rounding of the dumped k and v."""
    s = synth.ModelShape(1, 128, 4, 2, 32, 256, 300, 1e-5, 1e4, True)
    m = synth.make_model(s)
    orc = oracle.Oracle(s, m, "f64")
    P, tok, d, h2 = 37, 77, s.head_dim, s.head_dim // 2
    k, v = synth.alloc_kv(s, 1, 48)
    k[:, 0, :, :P] = synth.normal_bf16((1, s.n_kv_heads, P, d), synth.key(96, 4), 1.0)
    v[:, 0, :, :P] = synth.normal_bf16((1, s.n_kv_heads, P, d), synth.key(96, 5), 1.0)
    _, dump = orc.decode_step(k, v, 0, tok, P, dump=True)
    L = {n: widen(m["layers"][0][n]) for n in synth.LAYER_TENSORS}
    a = _np_rms(widen(m["embed"][tok]), L["attn_norm"], s.rms_eps)
    np.testing.assert_allclose(dump["v"][0], L["wv"] @ a, rtol=1e-12, atol=1e-15)
    want_angle = P * s.rope_theta ** (-2.0 * np.arange(h2) / d)
    for name, W in (("q", L["wq"]), ("k", L["wk"])):
        raw = (W @ a).reshape(-1, d)
        got = dump[name][0].reshape(-1, d)
        r0, r1, g0, g1 = raw[:, :h2], raw[:, h2:], got[:, :h2], got[:, h2:]
        np.testing.assert_allclose(np.hypot(g0, g1), np.hypot(r0, r1), rtol=1e-12)
        turn = np.angle((g0 + 1j * g1) / (r0 + 1j * r1))
        diff = np.angle(np.exp(1j * (turn - want_angle[None, :])))
        assert np.max(np.abs(diff)) < 1e-9, name
    for g in range(s.n_kv_heads):
        kb = [oracle.real_to_bf16(float(x)) for x in dump["k"][0].reshape(-1, d)[g]]
        vb = [oracle.real_to_bf16(float(x)) for x in dump["v"][0].reshape(-1, d)[g]]
        assert list(k[0, 0, g, P]) == kb and list(v[0, 0, g, P]) == vb


def test_gqa_contiguous_groups():
    """KV head 0 holds V = +1, KV head 1 holds V = -1 at every earlier
    position; with contiguous grouping query heads 0,1 read head 0 and heads
    2,3 read head 1 (an h % n_kv mapping would mix them)."""
    s = synth.TINY
    m = synth.make_model(s)
    orc = oracle.Oracle(s, m, "f64")
    P = 60
    k, v = synth.alloc_kv(s, 1, 64)
    k[:, 0, :, :P, :] = synth.normal_bf16((s.n_layers, s.n_kv_heads, P, s.head_dim), synth.key(96, 1), 1.0)
    v[:, 0, 0, :P, :] = bf16(1.0)
    v[:, 0, 1, :P, :] = bf16(-1.0)
    _, dump = orc.decode_step(k, v, 0, 5, P, dump=True)
    d = s.head_dim
    for l in range(s.n_layers):
        heads = dump["attn"][l].reshape(s.n_q_heads, d)
        assert np.all(heads[0] > 0.5) and np.all(heads[1] > 0.5)
        assert np.all(heads[2] < -0.5) and np.all(heads[3] < -0.5)


def test_gqa_with_one_query_head_per_kv_head_is_mha():
    """n_kv = n_q: each query head attends over its own KV head only."""
    s = synth.ModelShape(1, 128, 4, 4, 32, 256, 200, 1e-5, 1e4, True)
    m = synth.make_model(s)
    orc = oracle.Oracle(s, m, "f64")
    P = 9
    k, v = synth.alloc_kv(s, 1, 16)
    k[:, 0, :, :P] = synth.normal_bf16((1, 4, P, 32), synth.key(96, 2), 1.0)
    v[:, 0, :, :P] = synth.normal_bf16((1, 4, P, 32), synth.key(96, 3), 1.0)
    _, dump = orc.decode_step(k, v, 0, 7, P, dump=True)
    q = dump["q"][0].reshape(4, 32)
    for h in range(4):
        o = oracle.attention_head(q[h], k[0, 0, h, :P + 1], v[0, 0, h, :P + 1], "f64")
        np.testing.assert_array_equal(dump["attn"][0].reshape(4, 32)[h], o)


def test_decode_writes_only_its_row(tiny_model):
    s = synth.TINY
    orc = oracle.Oracle(s, tiny_model, "f64")
    k, v = _tiny_kv(batch=2, max_seq=32)
    k0, v0 = k.copy(), v.copy()
    orc.decode_step(k, v, 1, 11, 5)
    changed = np.argwhere(k != k0)
    assert set(map(tuple, changed[:, [1, 3]].tolist())) == {(1, 5)}
    changedv = np.argwhere(v != v0)
    assert set(map(tuple, changedv[:, [1, 3]].tolist())) == {(1, 5)}


def test_bad_arguments_rejected(tiny_model):
    s = synth.TINY
    orc = oracle.Oracle(s, tiny_model, "f64")
    k, v = _tiny_kv()
    with pytest.raises(ValueError):
        orc.decode_step(k, v, 0, s.vocab, 0)
    with pytest.raises(ValueError):
        orc.decode_step(k, v, 0, 0, -1)
