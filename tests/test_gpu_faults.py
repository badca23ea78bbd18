"""Failure detection on the GPU without faulting it: a plan whose test hook
drops one producer instruction makes a dependency impossible; the bounded
device wait must give up after its (short) limit, report MK_ERR_TIMEOUT via
mk_get_status, let every CTA exit, and leave the engine usable."""
import numpy as np
import pytest
import torch

import decode_megakernel_interpreter_b200 as mk
from decode_megakernel_interpreter_b200 import harness
import synth
from gpu_common import HostSetup

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("exec_kw", [dict(), dict(sched="dynamic"), dict(sched="event")],
                         ids=["static", "dynamic", "event"])
def test_timeout_is_reported_and_engine_recovers(exec_kw):
    s = synth.TINY
    hs = HostSetup(s, 1, 80)
    hs.fill_prefix([40])
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, 1, 80)
    eng.plan(debug_drop_producer=True, wait_timeout_ns=50_000_000, **exec_kw)
    t = torch.tensor([3], dtype=torch.int32, device="cuda")
    p = torch.tensor([40], dtype=torch.int32, device="cuda")
    nxt = torch.empty(1, dtype=torch.int32, device="cuda")
    logits = torch.empty(1, s.vocab, device="cuda")
    eng.decode_step(t, p, logits, nxt)
    assert eng.status() == mk.MK_ERR_TIMEOUT
    assert eng.status() == mk.MK_OK  # cleared
    # a correct plan on the same handle works again
    eng.plan(**exec_kw)
    eng.decode_step(t, p, logits, nxt)
    assert eng.status() == mk.MK_OK
    ol = hs.orc.decode_step(hs.k, hs.v, 0, 3, 40)
    np.testing.assert_allclose(logits[0].cpu().numpy(), ol, atol=2e-2, rtol=1e-2)
    eng.close()


def test_step_before_plan_is_rejected():
    s = synth.TINY
    hs = HostSetup(s, 1, 16)
    dev = harness.upload_model(hs.model, s.tied)
    kc, vc = harness.upload_kv(hs.k, hs.v)
    eng = harness.make_engine(s, dev, kc, vc, 1, 16)
    t = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = mk.mk_decode_step(eng.h, t.data_ptr(), t.data_ptr(), None, t.data_ptr(), None)
    assert rc == mk.MK_ERR_NOT_PLANNED
    with pytest.raises(mk.MkError):
        eng.plan(batch=2)
    eng.close()
