"""Tensor-parallel group (mk_tp_*), emulated on one GPU, against the CPU
oracle.

Rank r of n holds its query / KV heads, FFN columns and vocabulary rows; the
O and down projections store their partial sums into every rank's buffers and
the consumers sum the ranks' partials in rank order, so the result differs
from the single-GPU step only in the order of those sums.  Per step: logits
within the logit tolerance, the greedy id the oracle's (near-tie rule), and
every K/V row (all heads: each written by its rank) within one bf16 ulp plus
the fp32 dot-product bound.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import decode_megakernel_interpreter_b200 as mk
from decode_megakernel_interpreter_b200 import harness
import synth
from gpu_common import NORM_SIGMA, HostSetup, StepCheck, kv_row_mismatch


def llama1b_2layer():
    return dataclasses.replace(synth.WORKLOADS["llama1b"].shape, n_layers=2)


@pytest.mark.gpu
@pytest.mark.parametrize("n_ranks,norm_sigma", [(2, 0.0), (4, 0.0), (8, 0.0), (2, NORM_SIGMA)],
                         ids=["tp2", "tp4", "tp8", "tp2_seeded_norms"])
def test_llama1b_shape_tp_group(n_ranks, norm_sigma):
    s = llama1b_2layer()
    max_seq = 160
    hs = HostSetup(s, 1, max_seq, synth.make_model(s, norm_sigma=norm_sigma))
    hs.fill_prefix([100])
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = mk.TpEngine(s, dev, kc, vc, 1, max_seq, n_ranks)
    try:
        eng.plan(batch=1)
        tokens = torch.zeros(1, dtype=torch.int32, device="cuda")
        pos = torch.zeros(1, dtype=torch.int32, device="cuda")
        logits = torch.empty(1, s.vocab, dtype=torch.float32, device="cuda")
        nxt = torch.empty(1, dtype=torch.int32, device="cuda")
        tok, p = 17, 100
        chk = StepCheck()
        for step in range(5):
            tokens.fill_(tok)
            pos.fill_(p)
            eng.decode_step(tokens, pos, logits, nxt)
            assert eng.status() == mk.MK_OK
            gl = logits[0].cpu().numpy()
            gn = int(nxt.item())
            assert gn == int(np.argmax(gl)), "next token must be the first maximal logit"
            ol, bk, bv = hs.decode(0, tok, p)
            chk.check(gl, ol, gn, f"step {step}")
            mk_k = kv_row_mismatch(harness.kv_row_to_host(kc, 0, p), hs.k[:, 0, :, p], bk)
            mk_v = kv_row_mismatch(harness.kv_row_to_host(vc, 0, p), hs.v[:, 0, :, p], bv)
            assert not mk_k, f"step {step}: K row: {mk_k}"
            assert not mk_v, f"step {step}: V row: {mk_v}"
            tok, p = gn, p + 1
        assert chk.id_mismatches <= chk.near_ties
    finally:
        eng.close()


@pytest.mark.gpu
def test_tp_group_rejects_unsplittable_shapes_and_options():
    s = llama1b_2layer()
    hs = HostSetup(s, 1, 64)
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    with pytest.raises(mk.MkError):
        mk.TpEngine(s, dev, kc, vc, 1, 64, 16)  # 16 ranks: 8 KV heads do not split
    eng = mk.TpEngine(s, dev, kc, vc, 1, 64, 2)
    try:
        for kw in (dict(batch=1, sched="dynamic"), dict(batch=1, exec_mode="per_op"), dict(batch=1, trace=True)):
            with pytest.raises(mk.MkError):
                eng.plan(**kw)
        nxt = torch.empty(1, dtype=torch.int32, device="cuda")
        with pytest.raises(mk.MkError):  # not planned
            eng.decode_step(nxt, nxt, None, nxt)
    finally:
        eng.close()


def test_tp_create_argument_checks_without_a_gpu():
    """Rank counts and shapes are checked before any CUDA call."""
    cfg = mk.make_config(synth.TINY, 1, 64)
    lw = (mk.mk_layer_weights * cfg.n_layers)()
    for i in range(cfg.n_layers):
        for n, _ in mk.mk_layer_weights._fields_:
            setattr(lw[i], n, 4096)
    w = mk.mk_weights(4096, None, 4096, lw)
    kv = mk.mk_kv_cache(4096, 4096)
    g = ctypes.c_void_p()
    L = mk.load()
    for n in (0, 1, 3, 16):
        assert L.mk_tp_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(kv), n, ctypes.byref(g)) == \
            mk.MK_ERR_INVALID_ARG
    assert L.mk_tp_create(None, ctypes.byref(w), ctypes.byref(kv), 2, ctypes.byref(g)) == mk.MK_ERR_INVALID_ARG
    shape = dataclasses.replace(synth.TINY, n_kv_heads=1, n_q_heads=4)
    cfg1 = mk.make_config(shape, 1, 64)
    assert L.mk_tp_create(ctypes.byref(cfg1), ctypes.byref(w), ctypes.byref(kv), 2, ctypes.byref(g)) == \
        mk.MK_ERR_UNSUPPORTED_SHAPE
