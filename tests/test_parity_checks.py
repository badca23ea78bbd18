"""The GPU parity checks themselves, exercised on the CPU: an fp32
implementation of the step (the oracle's fp32 twin) must pass them against
the fp64 oracle, and planted mistakes in its outputs must fail them."""
import numpy as np
import pytest

import oracle
import synth
from gpu_common import NORM_SIGMA, HostSetup, StepCheck, kv_row_mismatch


@pytest.fixture(scope="module")
def tiny_gamma():
    s = synth.TINY
    return s, synth.make_model(s, norm_sigma=NORM_SIGMA)


def _twin_steps(s, model, steps=6):
    """(fp64 host setup, fp32 twin caches, logits, ids) over `steps` greedy steps."""
    w = synth.WORKLOADS["tiny"]
    hs = HostSetup(s, 1, 96, model)
    prompt = synth.prompt_tokens(w)
    last = hs.prefill_prompt(prompt)
    k32, v32 = hs.k.copy(), hs.v.copy()
    o32 = oracle.Oracle(s, model, "f32")
    tok, pos = int(np.argmax(last)), len(prompt)
    out = []
    for _ in range(steps):
        l32 = o32.decode_step(k32, v32, 0, tok, pos)
        l64, bk, bv = hs.decode(0, tok, pos)
        out.append((tok, pos, l32, l64, bk, bv))
        tok, pos = int(np.argmax(l32)), pos + 1
    return hs, k32, v32, out


def test_fp32_twin_passes_the_parity_checks(tiny_gamma):
    s, model = tiny_gamma
    hs, k32, v32, out = _twin_steps(s, model)
    chk = StepCheck()
    for i, (tok, pos, l32, l64, bk, bv) in enumerate(out):
        chk.check(l32.astype(np.float32), l64, int(np.argmax(l32)), f"step {i}")
        assert kv_row_mismatch(k32[:, 0, :, pos], hs.k[:, 0, :, pos], bk) == ""
        assert kv_row_mismatch(v32[:, 0, :, pos], hs.v[:, 0, :, pos], bv) == ""
    assert chk.id_mismatches == 0 and chk.max_abs < 1e-3


def test_planted_kv_and_id_mistakes_fail(tiny_gamma):
    s, model = tiny_gamma
    hs, k32, v32, out = _twin_steps(s, model, steps=2)
    tok, pos, l32, l64, bk, bv = out[-1]
    d = s.head_dim
    # K row of the wrong position, un-rotated halves swapped, sign flipped
    assert kv_row_mismatch(k32[:, 0, :, pos - 1], hs.k[:, 0, :, pos], bk)
    swapped = np.concatenate([k32[:, 0, :, pos, d // 2:], k32[:, 0, :, pos, :d // 2]], axis=-1)
    assert kv_row_mismatch(np.ascontiguousarray(swapped), hs.k[:, 0, :, pos], bk)
    assert kv_row_mismatch(k32[:, 0, :, pos] ^ np.uint16(0x8000), hs.k[:, 0, :, pos], bk)
    # a V row scaled by 1.3 (e.g. a norm weight applied twice)
    v13 = synth.bf16_bits_to_f32(v32[:, 0, :, pos]) * np.float32(1.3)
    v13b = (v13.view(np.uint32) >> 16).astype(np.uint16)
    assert kv_row_mismatch(v13b, hs.v[:, 0, :, pos], bv)
    # a greedy id that is not the oracle's argmax outside a near tie
    chk = StepCheck()
    wrong = int(np.argsort(l64)[-2])
    with pytest.raises(AssertionError):
        chk.check(l64.astype(np.float32), l64, wrong, "planted")
    # logits of a model that ignores the norm weights
    unit = synth.make_model(s)
    hs_u = HostSetup(s, 1, 96, unit)
    w = synth.WORKLOADS["tiny"]
    hs_u.prefill_prompt(synth.prompt_tokens(w))
    lu = hs_u.orc.decode_step(hs_u.k, hs_u.v, 0, out[0][0], out[0][1])
    with pytest.raises(AssertionError):
        StepCheck().check(lu.astype(np.float32), out[0][3], int(np.argmax(lu)), "unit norms")
