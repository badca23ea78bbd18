"""The plan cost model (mk_host_plan_estimate): the CTA-wave approximation
and the S(b) > F comparison of the "One Megakernel is Not Enough" digest,
applied to this build's plans.  Checked here for the properties the model
must have whatever its constants: bytes floor, monotonicity, waves, the
effect of each parameter, and agreement with the orderings measured on the
B200."""
import ctypes

import pytest

import decode_megakernel_interpreter_b200 as mk
import synth


def cfg_for(name, max_batch=1, extra=64):
    w = synth.WORKLOADS[name]
    return mk.make_config(w.shape, max_batch, int(w.lengths().max()) + w.steps + extra)


def est(name, ctx=None, params=None, max_batch=1, num_ctas=148, **kw):
    w = synth.WORKLOADS[name]
    cfg = cfg_for(name, max_batch)
    return mk.mk_host_plan_estimate(cfg, mk.plan_opts(**kw), num_ctas, w.context if ctx is None else ctx, params)


def test_defaults_roundtrip():
    p = mk.mk_cost_params_default()
    assert p.sm_gbs > 0 and p.ring_pages >= 1 and p.exchange_us > 0 and p.conv_ctas == 0


def test_floor_is_the_plans_bytes_at_the_sm_bandwidth():
    """hbm_floor = (weight pages + K/V pages of the plan) x 16 KiB at every
    SM's bandwidth, and the step can never beat it."""
    w = synth.WORKLOADS["llama1b"]
    cfg = cfg_for("llama1b")
    *_, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=1), 148)
    e = est("llama1b", batch=1)
    p = mk.mk_cost_params_default()
    s = w.shape
    # K/V pages: every split's cached positions in 64-position pages (d = 64)
    kv_pages = 0
    n, S = w.context + 1, info.kv_splits
    chunk = -(-n // S)
    for sp in range(S):
        start = min(n, sp * chunk)
        cached = max(0, min(min(n, start + chunk), w.context) - start)
        kv_pages += -(-cached // (16384 // (4 * s.head_dim)))
    kv_pages *= s.n_layers * s.n_kv_heads
    weight_pages = -(-info.weight_bytes_per_step // 16384)
    floor = (weight_pages + kv_pages) * 16384 / (p.sm_gbs * 1e3 * 148)
    assert e.hbm_floor_us == pytest.approx(floor, rel=2e-3)
    assert e.step_us > e.hbm_floor_us


def test_slower_exchanges_and_compute_cost_more():
    base = est("llama1b", batch=1)
    p = mk.mk_cost_params_default()
    p.exchange_us *= 2
    assert est("llama1b", params=p, batch=1).step_us > base.step_us
    p = mk.mk_cost_params_default()
    p.page_us *= 4  # compute slower than the page stream
    assert est("llama1b", params=p, batch=1).step_us > base.step_us
    p = mk.mk_cost_params_default()
    p.sm_gbs /= 2
    e = est("llama1b", params=p, batch=1)
    assert e.hbm_floor_us == pytest.approx(2 * base.hbm_floor_us, rel=1e-6) and e.step_us > base.step_us


def test_longer_context_costs_more():
    """More K/V pages per split: a longer step (at 512 and 1024 positions
    every one of 18 splits still fits one page: same pages, same estimate)."""
    a = est("llama1b_8k", ctx=8192, batch=1, kv_splits=18)
    b = est("llama1b_8k", ctx=1024, batch=1, kv_splits=18)
    assert a.step_us > b.step_us and a.hbm_floor_us > b.hbm_floor_us
    c = est("llama1b", ctx=512, batch=1, kv_splits=18)
    d = est("llama1b", ctx=1024, batch=1, kv_splits=18)
    assert c.step_us == pytest.approx(d.step_us) and c.hbm_floor_us == pytest.approx(d.hbm_floor_us)


def test_cta_waves_of_the_conventional_path():
    """ceil(g / W): with half the CTAs every full stage takes two waves."""
    full = est("llama1b", batch=1)
    p = mk.mk_cost_params_default()
    p.conv_ctas = 74
    half = est("llama1b", params=p, batch=1)
    assert half.step_us == pytest.approx(full.step_us)  # the megakernel keeps its CTAs
    assert half.per_op_us > 1.5 * full.per_op_us - 16 * 5 * (p.launch_us + p.exchange_us)


def test_persistent_kernel_pays_at_batch_1_and_16():
    """S(b) = per-op - megakernel > 0 at batch 1 and 16 (measured on the B200:
    2755 vs 673 us and 10339 vs 6869 us per step)."""
    assert est("llama1b", batch=1).savings_us > 0
    assert est("llama1b_b16", max_batch=16, ctx=2336, batch=16).savings_us > 0


def test_tensor_cores_pay_at_batch_16():
    """The ordering measured on the B200 at 16 sequences: tensor cores
    (6.87 ms) beat CUDA cores (9.77 ms) for gate/up, down and the LM head."""
    tc = est("llama1b_b16", max_batch=16, ctx=2336, batch=16)
    cc = est("llama1b_b16", max_batch=16, ctx=2336, batch=16, use_tcgen05=-1)
    assert tc.step_us < cc.step_us


def test_dynamic_queue_is_refused():
    with pytest.raises(mk.MkError):
        est("llama1b", batch=1, sched="dynamic")


def test_bad_arguments():
    cfg = cfg_for("tiny")
    out = mk.mk_cost_estimate()
    L = mk.load()
    assert L.mk_host_plan_estimate(ctypes.byref(cfg), None, 0, 10, None, ctypes.byref(out), None, 0) == \
        mk.MK_ERR_INVALID_ARG
    assert L.mk_host_plan_estimate(ctypes.byref(cfg), None, 8, cfg.max_seq, None, ctypes.byref(out), None, 0) == \
        mk.MK_ERR_INVALID_ARG
    assert L.mk_host_plan_estimate(ctypes.byref(cfg), None, 8, 10, None, None, None, 0) == mk.MK_ERR_INVALID_ARG


@pytest.mark.parametrize("name,ctx,splits,measured", [("llama1b", 1088, 18, 673), ("llama1b_8k", 8224, 18, 851),
                                                      ("llama8b", 2064, 18, 3191), ("llama1b_b16", 1980, 4, 6933)])
def test_defaults_reproduce_the_measured_steps(name, ctx, splits, measured):
    """The default parameters are fitted to B200 measurements of these plans
    (CUDA events, SM clock 1965 MHz): the estimates stay within 10 %."""
    w = synth.WORKLOADS[name]
    e = est(name, ctx=ctx, max_batch=w.batch, batch=w.batch, kv_splits=splits)
    assert abs(e.step_us / measured - 1) < 0.10


def test_per_op_path_estimate_matches_the_graph_replay():
    """The conventional path replayed as a CUDA graph measured 2983 us per
    step on the Llama-1B shape at context 1024 (81 launches)."""
    e = est("llama1b", ctx=1088, batch=1, kv_splits=18)
    assert abs(e.per_op_us / 2983 - 1) < 0.10
