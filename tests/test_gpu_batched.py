"""Batched decode on the Llama-1B shape: 16 independent sequences with their
own KV lengths (uniform in [512, 4096]) share each weight page of a step.
Every sequence is checked against the oracle, and the execution modes agree
bit for bit."""
import numpy as np
import pytest
import torch

import decode_megakernel_interpreter_b200 as mk
from decode_megakernel_interpreter_b200 import harness
import synth
from gpu_common import NORM_SIGMA, HostSetup, StepCheck, kv_row_mismatch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def b16():
    w = synth.WORKLOADS["llama1b_b16"]
    lengths = w.lengths()
    model = synth.make_model(w.shape)
    return w, lengths, model


@pytest.fixture(scope="module")
def b16_norms(b16):
    w, lengths, model = b16
    return w, lengths, synth.with_norms(model, w.shape, NORM_SIGMA)


def _engine(w, lengths, model, plan_kw, steps):
    # room for every step's K/V row of the longest sequence
    hs = HostSetup(w.shape, w.batch, int(lengths.max()) + steps + 2, model)
    hs.fill_prefix(lengths)
    dev = harness.upload_model(hs.model, w.shape.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(w.shape, dev, kc, vc, w.batch, hs.max_seq)
    eng.plan(batch=w.batch, **plan_kw)
    return hs, eng, kc, vc


def _run(w, lengths, model, steps, plan_kw, check_oracle):
    hs, eng, kc, vc = _engine(w, lengths, model, plan_kw, steps)
    B = w.batch
    assert eng.info.kernel_variant == 1  # batched plans run a specialised build
    tok = [int(t) for t in synth.first_tokens(w)]
    pos = [int(p) for p in lengths]
    tokens = torch.empty(B, dtype=torch.int32, device="cuda")
    positions = torch.empty(B, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, w.shape.vocab, dtype=torch.float32, device="cuda")
    nxt = torch.empty(B, dtype=torch.int32, device="cuda")
    out = []
    chk = StepCheck()
    try:
        for step in range(steps):
            tokens.copy_(torch.tensor(tok, dtype=torch.int32))
            positions.copy_(torch.tensor(pos, dtype=torch.int32))
            eng.decode_step(tokens, positions, logits, nxt)
            rc = eng.status()
            assert rc == mk.MK_OK, (rc, mk.mk_get_error_detail(eng.h))
            gl = logits.cpu().numpy()
            gn = nxt.cpu().numpy()
            for b in range(B):
                assert int(gn[b]) == int(np.argmax(gl[b])), f"seq {b}: next token must be the first maximal logit"
            if check_oracle:
                for b in range(B):
                    ol, bk, bv = hs.decode(b, tok[b], pos[b])
                    chk.check(gl[b], ol, int(gn[b]), f"step {step} seq {b}")
                    mk_k = kv_row_mismatch(harness.kv_row_to_host(kc, b, pos[b]), hs.k[:, b, :, pos[b]], bk)
                    mk_v = kv_row_mismatch(harness.kv_row_to_host(vc, b, pos[b]), hs.v[:, b, :, pos[b]], bv)
                    assert not mk_k, f"step {step} seq {b}: K row: {mk_k}"
                    assert not mk_v, f"step {step} seq {b}: V row: {mk_v}"
            out.append(gl.copy())
            tok = [int(t) for t in gn]
            pos = [p + 1 for p in pos]
    finally:
        eng.close()
    if check_oracle:
        from test_gpu_parity import log_parity
        log_parity("batched", chk.record(), plan_kw)
        assert chk.id_mismatches <= chk.near_ties
    return out


def test_llama1b_batch16_matches_oracle(b16):
    """All 16 sequences free-running for 8 greedy steps."""
    w, lengths, model = b16
    _run(w, lengths, model, 8, dict(), check_oracle=True)


@pytest.mark.parametrize("kw", [dict(), dict(tensor_qkv_o=True)], ids=["default", "tensor_qkv_o"])
def test_llama1b_batch16_norm_weights(b16_norms, kw):
    """Seeded norm weights on both batched builds: the tensor-core operands
    carry x * gamma as bf16 hi/lo, so a wrong gamma there shows in every
    sequence's logits."""
    w, lengths, model = b16_norms
    _run(w, lengths, model, 2, kw, check_oracle=True)


def test_llama1b_batch16_modes_agree(b16):
    w, lengths, model = b16
    ref = _run(w, lengths, model, 2, dict(), check_oracle=False)
    for kw in (dict(exec_mode="per_op"), dict(sched="dynamic"), dict(sched="event")):
        got = _run(w, lengths, model, 2, kw, check_oracle=False)
        for a, b in zip(ref, got):
            np.testing.assert_array_equal(a, b)


def test_llama1b_batch16_tensor_qkv_o_matches_oracle(b16):
    """QKV (with RoPE and the K/V append) and the O projection as tensor-core
    tiles: every sequence against the oracle, and the per-op path agrees bit
    for bit."""
    w, lengths, model = b16
    ref = _run(w, lengths, model, 2, dict(tensor_qkv_o=True), check_oracle=True)
    got = _run(w, lengths, model, 2, dict(tensor_qkv_o=True, exec_mode="per_op"), check_oracle=False)
    for a, b in zip(ref, got):
        np.testing.assert_array_equal(a, b)


def test_llama1b_batch16_cuda_cores_match_oracle(b16):
    """use_tcgen05 = -1: the same batched build with every matrix instruction
    on CUDA cores (the comparison the tensor-core path is adopted against)."""
    w, lengths, model = b16
    _run(w, lengths, model, 2, dict(use_tcgen05=-1), check_oracle=True)


def test_batched_plan_needs_a_batched_build():
    """Shapes without a batched build refuse batch > 1 (the tiny shape)."""
    s = synth.TINY
    hs = HostSetup(s, 2, 16)
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, 2, 16)
    with pytest.raises(mk.MkError):
        eng.plan(batch=2)
    eng.close()
