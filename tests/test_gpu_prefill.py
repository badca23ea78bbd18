"""GPU prefill (mk_prefill) against the CPU oracle.

Prompt tokens run through the persistent interpreter: one token per launch
with a batch-1 plan, or chunks of up to 16 tokens per launch with the batched
tensor-core plan, where token j of a chunk attends over the cache rows before
the chunk and the chunk's rows 0..j.  The oracle decodes the same tokens one
by one; every K/V row the prompt wrote must be within one bf16 ulp plus the
fp32 dot-product bound of the oracle's, the last token's logits within the
logit tolerance, its greedy id the oracle's (near-tie rule), and decoding must
then continue from the GPU-filled cache in step with the oracle.
"""
import dataclasses

import numpy as np
import pytest
import torch

import decode_megakernel_interpreter_b200 as mk
from decode_megakernel_interpreter_b200 import harness
import synth
from gpu_common import HostSetup, StepCheck, kv_row_mismatch

pytestmark = pytest.mark.gpu


def check_prompt(hs, kc, vc, b, prompt, pos0, gpu_logits, gpu_next, chk):
    """Oracle-decode the prompt at sequence b; compare every K/V row and the
    last token's logits and greedy id."""
    ol = None
    for j, t in enumerate(prompt):
        ol, bk, bv = hs.decode(b, int(t), pos0 + j)
        p = pos0 + j
        mk_k = kv_row_mismatch(harness.kv_row_to_host(kc, b, p), hs.k[:, b, :, p], bk)
        mk_v = kv_row_mismatch(harness.kv_row_to_host(vc, b, p), hs.v[:, b, :, p], bv)
        assert not mk_k, f"prompt token {j}: K row: {mk_k}"
        assert not mk_v, f"prompt token {j}: V row: {mk_v}"
    chk.check(gpu_logits, ol, gpu_next, "last prompt token")


def continue_decode(eng, hs, kc, vc, b, tok, pos, steps, chk):
    """Greedy decode of sequence b from the GPU-filled cache, step by step
    against the oracle (fed the GPU's tokens)."""
    s = hs.shape
    B = eng.opts.batch
    tokens = torch.zeros(B, dtype=torch.int32, device="cuda")
    posv = torch.zeros(B, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, s.vocab, dtype=torch.float32, device="cuda")
    nxt = torch.empty(B, dtype=torch.int32, device="cuda")
    for step in range(steps):
        tokens.fill_(tok)
        posv.fill_(pos)
        if B > 1:  # the other rows decode their own sequences at their own lengths
            posv.copy_(torch.tensor(hs.lengths_now, dtype=torch.int32))
            posv[b] = pos
        eng.decode_step(tokens, posv, logits, nxt)
        assert eng.status() == mk.MK_OK, mk.mk_get_error_detail(eng.h)
        gl = logits[b].cpu().numpy()
        gn = int(nxt[b].item())
        ol, bk, bv = hs.decode(b, tok, pos)
        chk.check(gl, ol, gn, f"decode step {step}")
        mk_k = kv_row_mismatch(harness.kv_row_to_host(kc, b, pos), hs.k[:, b, :, pos], bk)
        assert not mk_k, f"decode step {step}: K row: {mk_k}"
        tok, pos = gn, pos + 1


@pytest.mark.parametrize("sched", ["static", "dynamic", "event"])
def test_tiny_prompt_one_token_per_launch(sched):
    """The tiny configuration's 64-token prompt on an empty cache, batch-1
    plan (one launch per token; each scheduling mode), then 8 decode steps."""
    s = synth.TINY
    w = synth.WORKLOADS["tiny"]
    prompt = [int(t) for t in synth.prompt_tokens(w)]
    hs = HostSetup(s, 1, 96)
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, 1, 96)
    try:
        eng.plan(batch=1, sched=sched)
        toks = torch.tensor(prompt, dtype=torch.int32, device="cuda")
        logits = torch.empty(s.vocab, dtype=torch.float32, device="cuda")
        nxt = torch.empty(1, dtype=torch.int32, device="cuda")
        eng.prefill(0, toks, 0, logits, nxt)
        assert eng.status() == mk.MK_OK, mk.mk_get_error_detail(eng.h)
        gl = logits.cpu().numpy()
        gn = int(nxt.item())
        assert gn == int(np.argmax(gl))
        chk = StepCheck()
        check_prompt(hs, kc, vc, 0, prompt, 0, gl, gn, chk)
        continue_decode(eng, hs, kc, vc, 0, gn, len(prompt), 8, chk)
        assert chk.id_mismatches <= chk.near_ties
    finally:
        eng.close()


@pytest.mark.parametrize("n_prompt,pos0", [(40, 37), (16, 0), (1, 53)])
def test_llama1b_shape_chunked_prompt(n_prompt, pos0):
    """The Llama-1B shape (2 layers) with the batched tensor-core plan: a
    prompt of sequence 3 after a seeded prefix of pos0 rows runs in chunks of
    16 tokens (40 = 16 + 16 + 8; one chunk from an empty cache; a single
    token); the other sequences' rows are untouched; then 3 decode steps of
    all 16 sequences, sequence 3 checked against the oracle."""
    base = synth.WORKLOADS["llama1b"].shape
    s = dataclasses.replace(base, n_layers=2)
    B, max_seq = 16, 160
    hs = HostSetup(s, B, max_seq)
    lengths = [pos0 if b == 3 else 20 + 5 * b for b in range(B)]
    hs.fill_prefix(lengths)
    rng = np.random.default_rng(1000 + n_prompt)
    prompt = [int(t) for t in rng.integers(0, s.vocab, n_prompt)]
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, B, max_seq)
    try:
        eng.plan(batch=B)
        before = [harness.kv_row_to_host(kc, 2, p).copy() for p in range(pos0, pos0 + n_prompt)]
        toks = torch.tensor(prompt, dtype=torch.int32, device="cuda")
        logits = torch.empty(s.vocab, dtype=torch.float32, device="cuda")
        nxt = torch.empty(1, dtype=torch.int32, device="cuda")
        eng.prefill(3, toks, pos0, logits, nxt)
        assert eng.status() == mk.MK_OK, mk.mk_get_error_detail(eng.h)
        for p, row in zip(range(pos0, pos0 + n_prompt), before):
            np.testing.assert_array_equal(harness.kv_row_to_host(kc, 2, p), row)
        gl = logits.cpu().numpy()
        gn = int(nxt.item())
        assert gn == int(np.argmax(gl))
        chk = StepCheck()
        check_prompt(hs, kc, vc, 3, prompt, pos0, gl, gn, chk)
        hs.lengths_now = list(lengths)
        continue_decode(eng, hs, kc, vc, 3, gn, pos0 + n_prompt, 3, chk)
        assert chk.id_mismatches <= chk.near_ties
    finally:
        eng.close()


def test_llama8b_shape_prompt_second_sequence():
    """The Llama-8B shape (2 layers; the split-page build, head_dim 128) with a
    batch-1 plan on a two-sequence cache: an 8-token prompt of sequence 1,
    one token per launch; sequence 0's rows untouched."""
    base = synth.WORKLOADS["llama8b"].shape
    s = dataclasses.replace(base, n_layers=2)
    max_seq = 48
    hs = HostSetup(s, 2, max_seq)
    hs.fill_prefix([20, 12])
    rng = np.random.default_rng(88)
    prompt = [int(t) for t in rng.integers(0, s.vocab, 8)]
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, 2, max_seq)
    try:
        eng.plan(batch=1)
        assert eng.info.kernel_variant == 1  # the shape-specialised (split-page) build
        before = [harness.kv_row_to_host(kc, 0, p).copy() for p in range(12, 20)]
        toks = torch.tensor(prompt, dtype=torch.int32, device="cuda")
        logits = torch.empty(s.vocab, dtype=torch.float32, device="cuda")
        nxt = torch.empty(1, dtype=torch.int32, device="cuda")
        eng.prefill(1, toks, 12, logits, nxt)
        assert eng.status() == mk.MK_OK, mk.mk_get_error_detail(eng.h)
        for p, row in zip(range(12, 20), before):
            np.testing.assert_array_equal(harness.kv_row_to_host(kc, 0, p), row)
        gl = logits.cpu().numpy()
        gn = int(nxt.item())
        assert gn == int(np.argmax(gl))
        chk = StepCheck()
        check_prompt(hs, kc, vc, 1, prompt, 12, gl, gn, chk)
        assert chk.id_mismatches <= chk.near_ties
    finally:
        eng.close()


def test_prefill_rejects_bad_arguments():
    s = synth.TINY
    hs = HostSetup(s, 1, 40)
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, 1, 40)
    try:
        toks = torch.zeros(8, dtype=torch.int32, device="cuda")
        nxt = torch.empty(1, dtype=torch.int32, device="cuda")
        with pytest.raises(mk.MkError):  # not planned
            eng.prefill(0, toks, 0, None, nxt)
        eng.plan(batch=1)
        for seq, pos0 in ((1, 0), (-1, 0), (0, 33), (0, -1)):  # seq outside max_batch; past max_seq
            with pytest.raises(mk.MkError):
                eng.prefill(seq, toks, pos0, None, nxt)
        eng.plan(batch=1, exec_mode="per_op")
        with pytest.raises(mk.MkError):
            eng.prefill(0, toks, 0, None, nxt)
    finally:
        eng.close()
