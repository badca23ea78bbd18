"""mk_decode_step_noalloc against mk_decode_step.

The allocation-free entry point serves callers that cannot allocate device
memory when they run a step (its scratch is a fixed device array inside the
library, and it reads the weights in the caller's layout instead of a
repacked copy).  It must produce what the handle-based path produces: here,
on two calls in a row (the second one fed the first one's token at the next
position), the logits within the parity tolerance of the tests (they are in
fact expected to be identical), the same next tokens and the same KV rows.
This file sorts last so a failure here comes after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_megakernel_interpreter_b200 as mk
from decode_megakernel_interpreter_b200 import harness
import synth
from gpu_common import ATOL, RTOL

pytestmark = pytest.mark.gpu


def _setup(shape, max_seq, context):
    model = synth.make_model(shape)
    k, v = synth.alloc_kv(shape, 1, max_seq)
    synth.fill_kv_prefix(shape, k, v, [context])
    dev = harness.upload_model(model, shape.tied)
    return model, dev, k, v


def _abi_structs(shape, dev, kc, vc, max_seq):
    cfg = mk.make_config(shape, 1, max_seq)
    layers = (mk.mk_layer_weights * shape.n_layers)()
    for i, L in enumerate(dev["layers"]):
        for n, _ in mk.mk_layer_weights._fields_:
            setattr(layers[i], n, L[n].data_ptr())
    lm = dev["lm_head"]
    w = mk.mk_weights(dev["embed"].data_ptr(), lm.data_ptr() if lm is not None else None,
                      dev["final_norm"].data_ptr(), layers)
    kv = mk.mk_kv_cache(kc.data_ptr(), vc.data_ptr())
    return cfg, w, kv, layers


@pytest.mark.parametrize("name, context", [("tiny", 64), ("llama1b", 1024)])
def test_noalloc_matches_handle_path_on_two_calls(name, context):
    shape = synth.WORKLOADS[name].shape
    max_seq = context + 4
    model, dev, k, v = _setup(shape, max_seq, context)
    # two identical caches: one per path
    kc_a, vc_a = harness.upload_kv(k, v)
    kc_b, vc_b = harness.upload_kv(k, v)
    eng = harness.make_engine(shape, dev, kc_a, vc_a, 1, max_seq)
    eng.plan()
    cfg, w, kv, _keep = _abi_structs(shape, dev, kc_b, vc_b, max_seq)
    stream = torch.cuda.current_stream()
    tok = int(synth.first_tokens(synth.WORKLOADS[name])[0]) % shape.vocab
    t_a = torch.tensor([tok], dtype=torch.int32, device="cuda")
    t_b = t_a.clone()
    logits_a = torch.empty(1, shape.vocab, device="cuda")
    logits_b = torch.empty(1, shape.vocab, device="cuda")
    for call in range(2):
        pos = torch.tensor([context + call], dtype=torch.int32, device="cuda")
        eng.decode_step(t_a, pos, logits_a, t_a)  # next token fed back in place
        rc = mk.mk_decode_step_noalloc(cfg, w, kv, t_b.data_ptr(), pos.data_ptr(), logits_b.data_ptr(),
                                       t_b.data_ptr(), stream.cuda_stream)
        assert rc == mk.MK_OK, mk.mk_status_string(rc)
        torch.cuda.synchronize()
        assert eng.status() == mk.MK_OK
        la, lb = logits_a.cpu().numpy(), logits_b.cpu().numpy()
        assert np.all(np.abs(lb - la) <= ATOL + RTOL * np.abs(la)), f"call {call}"
        np.testing.assert_array_equal(lb, la)  # same kernels, same plan: identical
        assert int(t_b.item()) == int(t_a.item()) == int(np.argmax(la[0]))
        p = context + call
        np.testing.assert_array_equal(harness.kv_to_host(kc_b)[:, 0, :, p], harness.kv_to_host(kc_a)[:, 0, :, p])
        np.testing.assert_array_equal(harness.kv_to_host(vc_b)[:, 0, :, p], harness.kv_to_host(vc_a)[:, 0, :, p])
    # a further call with the same arguments takes no device memory: free
    # memory is unchanged across it (torch's caching allocator is not involved
    # either, since the call goes straight through the C ABI)
    pos = torch.tensor([context + 2], dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    rc = mk.mk_decode_step_noalloc(cfg, w, kv, t_b.data_ptr(), pos.data_ptr(), logits_b.data_ptr(), t_b.data_ptr(),
                                   stream.cuda_stream)
    assert rc == mk.MK_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    eng.close()


def test_noalloc_call_replays_from_a_cuda_graph():
    """After a first call (which uploads the plan and tables and
    synchronises), a call with the same arguments only enqueues device work:
    captured once in a CUDA graph, its replays at later positions (updated in
    place in the captured position buffer) give the handle path's results."""
    shape = synth.TINY
    context, max_seq = 64, 80
    model, dev, k, v = _setup(shape, max_seq, context)
    kc_a, vc_a = harness.upload_kv(k, v)
    kc_b, vc_b = harness.upload_kv(k, v)
    eng = harness.make_engine(shape, dev, kc_a, vc_a, 1, max_seq)
    eng.plan()
    cfg, w, kv, _keep = _abi_structs(shape, dev, kc_b, vc_b, max_seq)
    t_a = torch.tensor([7], dtype=torch.int32, device="cuda")
    t_b = t_a.clone()
    pos_a = torch.tensor([context], dtype=torch.int32, device="cuda")
    pos_b = pos_a.clone()
    logits_a = torch.empty(1, shape.vocab, device="cuda")
    logits_b = torch.empty(1, shape.vocab, device="cuda")
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):  # the first call: uploads, synchronises
        rc = mk.mk_decode_step_noalloc(cfg, w, kv, t_b.data_ptr(), pos_b.data_ptr(), logits_b.data_ptr(),
                                       t_b.data_ptr(), side.cuda_stream)
        assert rc == mk.MK_OK
    side.synchronize()
    eng.decode_step(t_a, pos_a, logits_a, t_a)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(logits_b.cpu().numpy(), logits_a.cpu().numpy())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        rc = mk.mk_decode_step_noalloc(cfg, w, kv, t_b.data_ptr(), pos_b.data_ptr(), logits_b.data_ptr(),
                                       t_b.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == mk.MK_OK
    for step in range(1, 4):
        pos_a.fill_(context + step)
        pos_b.fill_(context + step)
        graph.replay()
        eng.decode_step(t_a, pos_a, logits_a, t_a)
        torch.cuda.synchronize()
        assert eng.status() == mk.MK_OK
        np.testing.assert_array_equal(logits_b.cpu().numpy(), logits_a.cpu().numpy())
        assert int(t_b.item()) == int(t_a.item())
    del graph
    eng.close()


def test_noalloc_reports_device_side_errors():
    """A token id outside the vocabulary is clamped and reported by
    mk_noalloc_get_status; the next call clears it."""
    shape = synth.TINY
    context, max_seq = 40, 48
    model, dev, k, v = _setup(shape, max_seq, context)
    kc, vc = harness.upload_kv(k, v)
    cfg, w, kv, _keep = _abi_structs(shape, dev, kc, vc, max_seq)
    stream = torch.cuda.current_stream()
    pos = torch.tensor([context], dtype=torch.int32, device="cuda")
    nxt = torch.empty(1, dtype=torch.int32, device="cuda")
    bad = torch.tensor([shape.vocab + 5], dtype=torch.int32, device="cuda")
    rc = mk.mk_decode_step_noalloc(cfg, w, kv, bad.data_ptr(), pos.data_ptr(), None, nxt.data_ptr(), stream.cuda_stream)
    assert rc == mk.MK_OK
    code, detail = mk.mk_noalloc_get_status(stream.cuda_stream)
    assert code == mk.MK_ERR_DEVICE_INPUT, (code, detail)
    good = torch.tensor([3], dtype=torch.int32, device="cuda")
    rc = mk.mk_decode_step_noalloc(cfg, w, kv, good.data_ptr(), pos.data_ptr(), None, nxt.data_ptr(), stream.cuda_stream)
    assert rc == mk.MK_OK
    assert mk.mk_noalloc_get_status(stream.cuda_stream)[0] == mk.MK_OK


def test_noalloc_rejects_oversized_and_bad_arguments():
    shape = synth.TINY
    model, dev, k, v = _setup(shape, 16, 8)
    kc, vc = harness.upload_kv(k, v)
    t = torch.zeros(1, dtype=torch.int32, device="cuda")
    # a context so long that the RoPE table alone exceeds the fixed scratch
    cfg, w, kv, _keep = _abi_structs(shape, dev, kc, vc, 16)
    cfg.max_seq = 1 << 20
    rc = mk.mk_decode_step_noalloc(cfg, w, kv, t.data_ptr(), t.data_ptr(), None, t.data_ptr(), None)
    assert rc == mk.MK_ERR_UNSUPPORTED_SHAPE
    cfg.max_seq = 16
    cfg.max_batch = 2  # batch of this call must be 1
    assert mk.mk_decode_step_noalloc(cfg, w, kv, t.data_ptr(), t.data_ptr(), None, t.data_ptr(), None) == \
        mk.MK_ERR_UNSUPPORTED_SHAPE
    cfg.max_batch = 1
    assert mk.load().mk_decode_step_noalloc(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(kv), None, None, None,
                                            None, None) == mk.MK_ERR_INVALID_ARG
