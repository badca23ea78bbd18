"""GPU parity: the engine (through the C ABI) against the CPU oracle on the
same seeded inputs.

Per step: every logit within |gpu - oracle| <= 2e-2 + 1e-2 |oracle| (the
oracle is fed the GPU's own input token, so the two never drift apart); the
greedy id identical to the oracle's unless the oracle's top-2 margin is within
twice the step's measured logit error (then the GPU's id must be one of the
ids that error allows); next_tokens_out == argmax(logits_out) exactly; and the
K/V row written at the step's position within one bf16 ulp plus the fp32
dot-product error bound of the oracle's.  Several tests use seeded norm
weights ~N(1, 0.3) (distinct per norm and layer) so that the kernels' use of
them is checked too; the full-size configurations run free for tens of steps.
"""
import json
import os

import numpy as np
import pytest
import torch

import decode_megakernel_interpreter_b200 as mk
from decode_megakernel_interpreter_b200 import harness
import synth
from gpu_common import NORM_SIGMA, HostSetup, StepCheck, kv_row_mismatch

pytestmark = pytest.mark.gpu


def log_parity(name: str, rec: dict, plan_kw: dict):
    log = os.environ.get("MK_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", name), **rec,
                                "plan": {k: str(v) for k, v in plan_kw.items()}}) + "\n")


def run_parity(hs: HostSetup, first_token: int, first_pos: int, steps: int, plan_kw: dict, b=0,
               check_kv=True, dev=None):
    s = hs.shape
    if dev is None:
        dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, hs.batch, hs.max_seq)
    eng.plan(**plan_kw)
    tokens = torch.zeros(hs.batch, dtype=torch.int32, device="cuda")
    pos = torch.zeros(hs.batch, dtype=torch.int32, device="cuda")
    logits = torch.empty(hs.batch, s.vocab, dtype=torch.float32, device="cuda")
    nxt = torch.empty(hs.batch, dtype=torch.int32, device="cuda")
    tok, p = first_token, first_pos
    chk = StepCheck()
    stats = {"tokens": [], "logits": [], "kernel_variant": int(eng.info.kernel_variant)}
    try:
        for step in range(steps):
            tokens.fill_(tok)
            pos.fill_(p)
            eng.decode_step(tokens, pos, logits, nxt)
            rc = eng.status()
            assert rc == mk.MK_OK, (rc, mk.mk_get_error_detail(eng.h))
            gl = logits[b].cpu().numpy()
            gn = int(nxt[b].item())
            assert gn == int(np.argmax(gl)), "next token must be the first maximal logit"
            if check_kv:
                ol, bk, bv = hs.decode(b, tok, p)
            else:
                ol = hs.orc.decode_step(hs.k, hs.v, b, tok, p)
            chk.check(gl, ol, gn, f"step {step}")
            if check_kv:
                mk_k = kv_row_mismatch(harness.kv_row_to_host(kc, b, p), hs.k[:, b, :, p], bk)
                mk_v = kv_row_mismatch(harness.kv_row_to_host(vc, b, p), hs.v[:, b, :, p], bv)
                assert not mk_k, f"step {step}: K row: {mk_k}"
                assert not mk_v, f"step {step}: V row: {mk_v}"
            stats["tokens"].append(gn)
            stats["logits"].append(gl.copy())
            tok, p = gn, p + 1
    finally:
        eng.close()
    stats.update(chk.record())
    log_parity("run_parity", chk.record(), plan_kw)
    assert chk.id_mismatches <= chk.near_ties
    return stats


# ------------------------------------------------------------------ tiny

@pytest.fixture(scope="module")
def tiny_model():
    return synth.make_model(synth.TINY)


def tiny_setup(model, max_seq=96):
    w = synth.WORKLOADS["tiny"]
    hs = HostSetup(synth.TINY, 1, max_seq, model)
    prompt = synth.prompt_tokens(w)
    last = hs.prefill_prompt(prompt)
    return hs, int(np.argmax(last)), len(prompt)


@pytest.mark.parametrize("kw", [
    dict(),
    dict(exec_mode="per_op"),
    dict(exec_mode="per_op_graph"),
    dict(exec_mode="megakernel_generic"),
    dict(sched="dynamic"),
    dict(sched="event"),
    dict(sched="event", num_sms=3),
    dict(num_sms=3, kv_splits=7),
    dict(num_sms=1, kv_splits=1),
    dict(l2_prefetch_kb=256),
], ids=["mk", "per_op", "per_op_graph", "mk_generic", "dynamic", "event", "event3sm", "3sm", "1sm", "l2pf"])
def test_tiny_16_steps(tiny_model, kw):
    hs, tok, pos = tiny_setup(tiny_model)
    run_parity(hs, tok, pos, 16, kw)


def test_schedule_independence_bitwise(tiny_model):
    """Every row's dot product runs inside one page on one warp, so the plan's
    placement must not change a single bit (fixed kv_splits)."""
    outs = []
    for kw in (dict(kv_splits=4), dict(kv_splits=4, exec_mode="per_op"), dict(kv_splits=4, sched="dynamic"),
               dict(kv_splits=4, sched="event"), dict(kv_splits=4, num_sms=5)):
        hs, tok, pos = tiny_setup(tiny_model)
        outs.append(run_parity(hs, tok, pos, 4, kw))
    for o in outs[1:]:
        assert o["tokens"] == outs[0]["tokens"]
        for a, b in zip(o["logits"], outs[0]["logits"]):
            np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("kw", [dict(), dict(exec_mode="per_op"), dict(exec_mode="megakernel_generic")],
                         ids=["mk", "per_op", "mk_generic"])
def test_tiny_norm_weights(tiny_model, kw):
    """Seeded norm weights ~N(1, 0.3), distinct per norm and layer: a kernel
    that ignored them, swapped the attention and FFN norms, skipped the final
    norm or indexed gamma in the wrong layout would fail the logits."""
    model = synth.with_norms(tiny_model, synth.TINY, NORM_SIGMA)
    hs, tok, pos = tiny_setup(model)
    run_parity(hs, tok, pos, 16, kw)


def test_tiny_from_empty_cache(tiny_model):
    """Position 0: attention over the single current key."""
    hs = HostSetup(synth.TINY, 1, 32, tiny_model)
    run_parity(hs, 17, 0, 8, dict(kv_splits=5))


def test_tiny_last_position(tiny_model):
    hs, tok, pos = tiny_setup(tiny_model, max_seq=66)
    run_parity(hs, tok, pos, 2, dict())  # positions 64 and 65 = max_seq - 1


def test_ragged_vocab_and_untied_head():
    """vocab not a multiple of the rows per page: a partial last LM page."""
    s = synth.ModelShape(2, 256, 4, 2, 64, 512, 1000, 1e-5, 1e4, False)
    hs = HostSetup(s, 1, 48)
    hs.fill_prefix([30])
    run_parity(hs, 999, 30, 6, dict())


@pytest.mark.parametrize("norm_sigma", [0.0, NORM_SIGMA], ids=["unit_norms", "seeded_norms"])
def test_mha_and_head_dim_128(norm_sigma):
    s = synth.ModelShape(2, 512, 4, 4, 128, 2048, 2048, 1e-5, 5e5, True)
    hs = HostSetup(s, 1, 200, synth.make_model(s, norm_sigma=norm_sigma))
    hs.fill_prefix([150])
    run_parity(hs, 5, 150, 4, dict(kv_splits=6))


@pytest.mark.parametrize("norm_sigma", [0.0, NORM_SIGMA], ids=["unit_norms", "seeded_norms"])
def test_gqa_group_of_eight(norm_sigma):
    s = synth.ModelShape(1, 1024, 16, 2, 64, 4096, 3000, 1e-5, 1e4, True)
    hs = HostSetup(s, 1, 300, synth.make_model(s, norm_sigma=norm_sigma))
    hs.fill_prefix([257])
    run_parity(hs, 2999, 257, 3, dict())


def test_next_tokens_may_alias_tokens(tiny_model):
    """Feeding next_tokens_out back as tokens without a host round trip."""
    hs, tok, pos = tiny_setup(tiny_model)
    s = hs.shape
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, 1, hs.max_seq)
    eng.plan()
    buf = torch.tensor([tok], dtype=torch.int32, device="cuda")
    positions = [torch.tensor([pos + i], dtype=torch.int32, device="cuda") for i in range(6)]
    logits = torch.empty(1, s.vocab, device="cuda")
    got = []
    for i in range(6):
        eng.decode_step(buf, positions[i], logits, buf)
        got.append(buf.clone())
    assert eng.status() == mk.MK_OK
    eng.close()
    # the oracle, fed the GPU's own inputs, must agree with every pick
    # (no logits of these steps are kept: an id the oracle ranks below its
    # maximum by more than the logit tolerance is wrong)
    inp = tok
    for i in range(6):
        ol = hs.orc.decode_step(hs.k, hs.v, 0, inp, pos + i)
        out = int(got[i].item())
        assert ol[out] >= ol.max() - 2 * (2e-2 + 1e-2 * abs(float(ol.max())))
        inp = out


def test_bad_token_reported_and_clamped(tiny_model):
    hs, tok, pos = tiny_setup(tiny_model)
    s = hs.shape
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, 1, hs.max_seq)
    eng.plan()
    t = torch.tensor([s.vocab + 5], dtype=torch.int32, device="cuda")
    p = torch.tensor([pos], dtype=torch.int32, device="cuda")
    nxt = torch.empty(1, dtype=torch.int32, device="cuda")
    eng.decode_step(t, p, None, nxt)
    assert eng.status() == mk.MK_ERR_DEVICE_INPUT
    # the engine keeps working afterwards
    t.fill_(tok)
    eng.decode_step(t, p, None, nxt)
    assert eng.status() == mk.MK_OK
    eng.close()


def test_trace_records_every_instruction(tiny_model):
    hs, tok, pos = tiny_setup(tiny_model)
    s = hs.shape
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, 1, hs.max_seq)
    info = eng.plan(trace=True)
    t = torch.tensor([tok], dtype=torch.int32, device="cuda")
    p = torch.tensor([pos], dtype=torch.int32, device="cuda")
    nxt = torch.empty(1, dtype=torch.int32, device="cuda")
    eng.decode_step(t, p, None, nxt)
    assert eng.status() == mk.MK_OK
    tr = eng.trace()
    eng.close()
    assert tr.shape == (info.num_instructions, mk.MK_TRACE_WORDS)
    ops = tr[:, 7] & 0xFF
    assert set(ops.tolist()) == {1, 2, 3, 4, 5, 6}
    for a, b in ((0, 1), (1, 2), (2, 3), (3, 4), (5, 6)):
        assert np.all(tr[:, a] <= tr[:, b]), (a, b)
    assert np.all(tr[:, 4] - tr[:, 0] < 1_000_000_000)
    assert np.all(tr[:, 5] > 0)


# ------------------------------------------------------------------ full-size shapes

@pytest.fixture(scope="module")
def llama1b_model():
    return synth.make_model(synth.LLAMA_1B)


def test_llama1b_1024_context(llama1b_model):
    """The headline configuration, free-running for 32 greedy steps."""
    w = synth.WORKLOADS["llama1b"]
    hs = HostSetup(w.shape, 1, w.context + 40, llama1b_model)
    hs.fill_prefix(w.lengths())
    st = run_parity(hs, int(synth.first_tokens(w)[0]), w.context, 32, dict())
    print("llama1b", {k: st[k] for k in ("max_abs", "max_rel", "near_ties", "id_mismatches")})


def test_llama1b_1024_context_norm_weights(llama1b_model):
    w = synth.WORKLOADS["llama1b"]
    model = synth.with_norms(llama1b_model, w.shape, NORM_SIGMA)
    hs = HostSetup(w.shape, 1, w.context + 8, model)
    hs.fill_prefix(w.lengths())
    run_parity(hs, int(synth.first_tokens(w)[0]), w.context, 4, dict())


def test_llama1b_8k_context(llama1b_model):
    """Context 8192, free-running for 16 greedy steps."""
    w = synth.WORKLOADS["llama1b_8k"]
    hs = HostSetup(w.shape, 1, w.context + 20, llama1b_model)
    hs.fill_prefix(w.lengths())
    run_parity(hs, int(synth.first_tokens(w)[0]), w.context, 16, dict())


def test_llama1b_per_op_and_generic_match_megakernel(llama1b_model):
    """The shape-specialised interpreter (the default for this shape), the
    shape-generic one and the per-op launches compute bit-identical steps."""
    w = synth.WORKLOADS["llama1b"]
    outs = []
    for kw in (dict(), dict(exec_mode="per_op"), dict(exec_mode="megakernel_generic")):
        hs = HostSetup(w.shape, 1, w.context + 4, llama1b_model)
        hs.fill_prefix(w.lengths())
        outs.append(run_parity(hs, int(synth.first_tokens(w)[0]), w.context, 2, kw, check_kv=False))
    assert [o["kernel_variant"] for o in outs] == [1, 1, 0]
    for o in outs[1:]:
        for a, b in zip(outs[0]["logits"], o["logits"]):
            np.testing.assert_array_equal(a, b)


def test_llama8b_2048_context():
    """The 8B shape (untied head, head_dim 128): 4 free-running greedy steps
    with the configuration's unit norm weights, then 2 with seeded ones (same
    matrices on the device)."""
    w = synth.WORKLOADS["llama8b"]
    model = synth.make_model(w.shape)
    dev = harness.upload_model(model, w.shape.tied)
    hs = HostSetup(w.shape, 1, w.context + 8, model)
    hs.fill_prefix(w.lengths())
    run_parity(hs, int(synth.first_tokens(w)[0]), w.context, 4, dict(), dev=dev)
    gm = synth.with_norms(model, w.shape, NORM_SIGMA)
    hs = HostSetup(w.shape, 1, w.context + 8, gm)
    hs.fill_prefix(w.lengths())
    run_parity(hs, int(synth.first_tokens(w)[0]), w.context, 2, dict(), dev=harness.replace_norms(dev, gm))
