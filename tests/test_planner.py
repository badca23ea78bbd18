"""The host planner (no GPU): structure of the plans it emits and a host
simulation of the counter protocol (one CPU thread per CTA, real atomics,
random delays, version stamps on every buffer element)."""
import collections

import pytest

import decode_megakernel_interpreter_b200 as mk
import synth

OP = {v: k for k, v in mk.OP_NAMES.items()}
NOC = 0xFFFFFFFF


def cfg_for(name, max_batch=1, max_seq=None):
    w = synth.WORKLOADS[name]
    return mk.make_config(w.shape, max_batch, max_seq or (w.context + w.steps))


def check_structure(cfg, instrs, off, ln, num_ctas, dynamic=False):
    s = cfg
    Rh = 8192 // s.hidden
    Ro = 8192 // (s.n_q_heads * s.head_dim)
    KCd = s.ffn if s.ffn <= 2048 else 2048
    Rd = 8192 // KCd
    ndp = s.ffn // KCd
    P = {"qkv": (s.n_q_heads + 2 * s.n_kv_heads) * s.head_dim // Rh, "oproj": s.hidden // Ro,
         "gateup": s.ffn // (Rh // 2), "lmhead": -(-s.vocab // Rh)}
    by_seq = sorted(instrs, key=lambda i: i.seq)
    assert [i.seq for i in by_seq] == list(range(len(instrs)))
    # queues are subsequences of the global order and cover everything once
    if not dynamic:
        assert sum(ln) == len(instrs)
        for c in range(num_ctas):
            q = instrs[off[c]:off[c] + ln[c]]
            assert all(a.seq < b.seq for a, b in zip(q, q[1:]))
    # page coverage: every page of every stage exactly once
    cover = collections.Counter()
    for i in instrs:
        name = mk.OP_NAMES[i.op]
        if name in P or name == "down":
            key = (name, i.layer, i.c if name == "down" else 0)
            for pg in range(i.a, i.a + i.b):
                cover[key + (pg,)] += 1
    for l in range(s.n_layers):
        for name in ("qkv", "oproj", "gateup"):
            assert all(cover[(name, l, 0, pg)] == 1 for pg in range(P[name])), (name, l)
        for k in range(ndp):
            assert all(cover[("down", l, k, pg)] == 1 for pg in range(s.hidden // Rd))
    assert all(cover[("lmhead", s.n_layers, 0, pg)] == 1 for pg in range(P["lmhead"]))
    assert sum(cover.values()) == sum(cover[k] for k in cover)
    # waits: count == number of producers, all producers earlier
    prod = collections.defaultdict(list)
    for i in instrs:
        if i.sig_ctr != NOC:
            for k in range(i.sig_n):
                if i.op != OP["attn"] or i.b == 0:
                    prod[i.sig_ctr + k].append(i.seq)
                else:
                    prod.setdefault(i.sig_ctr + k, prod[i.sig_ctr + k])
    attn_last = collections.defaultdict(int)
    for i in instrs:
        if i.op == OP["attn"]:
            attn_last[i.sig_ctr] = max(attn_last[i.sig_ctr], i.seq)
    for i in instrs:
        if i.wait_ctr == NOC:
            continue
        assert len(prod[i.wait_ctr]) == i.wait_cnt, (mk.OP_NAMES[i.op], i.layer)
        assert max(prod[i.wait_ctr] + [attn_last.get(i.wait_ctr, -1)]) < i.seq
    # dependency chain of a layer: qkv waits for the previous layer's down
    first = {mk.OP_NAMES[i.op]: i for i in reversed(by_seq) if i.layer == 1}
    if s.n_layers > 1:
        assert first["qkv"].wait_ctr != NOC


@pytest.mark.parametrize("name", ["tiny", "llama1b", "llama1b_8k", "llama8b"])
@pytest.mark.parametrize("num_ctas", [148, 37, 5, 1])
def test_plan_structure(name, num_ctas):
    cfg = cfg_for(name)
    instrs, off, ln, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=1), num_ctas)
    check_structure(cfg, instrs, off, ln, num_ctas)
    assert info.num_instructions == len(instrs)
    s = synth.WORKLOADS[name].shape
    want = 2 * (s.n_params() - s.vocab * s.hidden * (1 if s.tied else 2) - s.hidden
                - s.n_layers * 2 * s.hidden) + 2 * s.vocab * s.hidden
    assert info.weight_bytes_per_step == want


@pytest.mark.parametrize("num_ctas", [148, 16])
def test_plan_structure_dynamic(num_ctas):
    cfg = cfg_for("llama1b")
    instrs, off, ln, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=1, sched="dynamic"), num_ctas)
    check_structure(cfg, instrs, off, ln, num_ctas, dynamic=True)
    assert [i.seq for i in instrs] == list(range(len(instrs)))


def test_static_plan_balances_bytes():
    cfg = cfg_for("llama1b")
    instrs, off, ln, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=1), 148)
    load = []
    for c in range(148):
        load.append(sum(i.b for i in instrs[off[c]:off[c] + ln[c]] if i.op not in (OP["attn"], 0)))
    assert max(load) <= min(load) * 1.03 + 8  # pages per CTA within ~3 %
    # at most one chunk per stage per CTA
    for c in range(148):
        keys = [(i.op, i.layer, i.c if i.op == OP["down"] else 0) for i in instrs[off[c]:off[c] + ln[c]]
                if i.op != OP["attn"]]
        assert len(keys) == len(set(keys))


SPLIT_CANDIDATES = (1, 2, 3, 4, 6, 8, 9, 12, 16, 18, 24, 32, 36, 48, 64)


@pytest.mark.parametrize("name", ["llama1b", "llama1b_8k", "llama1b_b16"])
def test_kv_splits_rule_cost_model_and_explicit(name):
    """0: the fixed rule (one attention item per CTA); -1: the candidate count
    with the least cost-model estimate at max_seq (ties: the smaller); > 0:
    as given.  mk_plan_info reports the model's estimate of the plan."""
    w = synth.WORKLOADS[name]
    cfg = cfg_for(name, max_batch=w.batch)
    B = w.batch
    *_, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=B), 148)
    items = B * w.shape.n_kv_heads
    rule = max(1, min(148 // items, cfg.max_seq // 32))
    if B > 1:
        rule = max(rule, min(3 * 148 // items, cfg.max_seq // 256))
    assert info.kv_splits == max(1, min(rule, 64))
    if B > 1:  # at the contexts the batched bench decodes (up to 4096 + its steps): 3 splits
        *_, info16 = mk.mk_host_plan(cfg_for(name, max_batch=B, max_seq=4200), mk.plan_opts(batch=B), 148)
        assert info16.kv_splits == 3
    est = lambda S: mk.mk_host_plan_estimate(cfg, mk.plan_opts(batch=B, kv_splits=S), 148, cfg.max_seq - 1).step_us
    assert info.estimated_step_us == round(est(info.kv_splits))
    *_, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=B, kv_splits=-1), 148)
    cands = [S for S in SPLIT_CANDIDATES if S <= max(1, min(64, cfg.max_seq // 32))]
    e = {}
    for S in cands:
        try:
            e[S] = est(S)
        except mk.MkError:  # a plan too large for one step
            pass
    best = min(e, key=lambda S: (e[S], S))
    assert info.kv_splits == best
    assert info.estimated_step_us == round(e[best])
    *_, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=B, kv_splits=5), 148)
    assert info.kv_splits == 5
    with pytest.raises(mk.MkError):
        mk.mk_host_plan(cfg, mk.plan_opts(batch=B, kv_splits=-2), 148)


@pytest.mark.parametrize("sched", ["static", "dynamic", "event"])
@pytest.mark.parametrize("num_ctas", [8, 3, 1])
def test_simulation_tiny(sched, num_ctas):
    cfg = cfg_for("tiny")
    err = mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=1, sched=sched, kv_splits=3), num_ctas, steps=3,
                                   seed=num_ctas)
    assert err == ""


@pytest.mark.parametrize("sched", ["static", "dynamic", "event"])
def test_simulation_llama1b_full_grid(sched):
    cfg = cfg_for("llama1b")
    err = mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=1, sched=sched), 148, steps=2, seed=7,
                                   timeout_ms=20000)
    assert err == ""


def test_simulation_detects_a_missing_producer():
    """The drop-a-producer test hook makes a wait impossible: the simulation
    must report it as a timeout instead of hanging."""
    cfg = cfg_for("tiny")
    err = mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=1, debug_drop_producer=True), 4, steps=1, seed=1,
                                   timeout_ms=300)
    assert "waited too long" in err


def test_simulation_event_queue_detects_a_missing_producer():
    """In the event-driven mode a dropped producer leaves its dependents out
    of the ready queue: the simulation reports the slot that is never filled."""
    cfg = cfg_for("tiny")
    err = mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=1, sched="event", debug_drop_producer=True), 4, steps=1,
                                   seed=1, timeout_ms=300)
    assert "never filled" in err


def test_event_plan_is_the_dynamic_order():
    """The event-driven plan holds the same instructions in the same
    topological order as the dynamic queue (only the claim order differs)."""
    cfg = cfg_for("llama1b")
    a, *_ = mk.mk_host_plan(cfg, mk.plan_opts(batch=1, sched="dynamic"), 148)
    b, *_ = mk.mk_host_plan(cfg, mk.plan_opts(batch=1, sched="event"), 148)
    assert [bytes(x) for x in a] == [bytes(x) for x in b]


def test_plan_rejects_bad_options():
    cfg = cfg_for("tiny")
    with pytest.raises(mk.MkError):
        o = mk.plan_opts(batch=1)
        o.sched_mode = 3
        mk.mk_host_plan(cfg, o, 8)
    with pytest.raises(mk.MkError):
        mk.mk_host_plan(cfg, mk.plan_opts(batch=2), 8)
    with pytest.raises(mk.MkError):
        mk.mk_host_plan(cfg, mk.plan_opts(batch=0), 8)


def test_batched_plan_uses_tensor_core_tiles():
    """Batched plans cover gate/up, down and the LM head in 128-row tiles
    (64 gate + 64 up rows for gate/up) and stream the same weight bytes as
    the batch-1 plan."""
    cfg1 = cfg_for("llama1b")
    *_, info1 = mk.mk_host_plan(cfg1, mk.plan_opts(batch=1), 148)
    cfg = cfg_for("llama1b_b16", max_batch=16)
    instrs, off, ln, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=16), 148)
    assert info.weight_bytes_per_step == info1.weight_bytes_per_step
    F, H, V = cfg.ffn, cfg.hidden, cfg.vocab
    for l in (0, cfg.n_layers - 1):
        gu = [i for i in instrs if i.op == OP["gateup"] and i.layer == l]
        assert sorted((i.a, i.a + i.b) for i in gu)[0][0] == 0
        assert sum(i.b for i in gu) == F // 64
        # the down projection in K pieces of 1024 columns, one 128-row tile per
        # instruction: every (piece, tile) once
        dn = [i for i in instrs if i.op == OP["down"] and i.layer == l]
        assert all(i.b == 1 for i in dn)
        assert sorted((i.c, i.a) for i in dn) == [(k, t) for k in range(F // 1024) for t in range(H // 128)]
    lm = [i for i in instrs if i.op == OP["lmhead"]]
    assert sum(i.b for i in lm) == -(-V // 128)
    err = mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=16), 148, steps=1, seed=5, timeout_ms=20000)
    assert err == ""


def test_batched_plan_tensor_qkv_o_tiles():
    """With tensor_qkv_o, QKV covers the [q; k; v] rows and the O projection
    the hidden rows in 128-row tiles, each tile once per layer; the weight
    bytes stay those of the batch-1 plan and the counter protocol holds."""
    cfg1 = cfg_for("llama1b")
    *_, info1 = mk.mk_host_plan(cfg1, mk.plan_opts(batch=1), 148)
    cfg = cfg_for("llama1b_b16", max_batch=16)
    opts = mk.plan_opts(batch=16, tensor_qkv_o=True)
    instrs, off, ln, info = mk.mk_host_plan(cfg, opts, 148)
    assert info.weight_bytes_per_step == info1.weight_bytes_per_step
    rows_qkv = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
    for l in range(cfg.n_layers):
        for op, n in (("qkv", rows_qkv // 128), ("oproj", cfg.hidden // 128)):
            spans = sorted((i.a, i.a + i.b) for i in instrs if i.op == OP[op] and i.layer == l)
            covered = [u for a, e in spans for u in range(a, e)]
            assert covered == list(range(n)), (op, l)
    # the default keeps them on CUDA cores, one page per unit
    instrs0, *_ = mk.mk_host_plan(cfg, mk.plan_opts(batch=16), 148)
    assert sum(i.b for i in instrs0 if i.op == OP["qkv"] and i.layer == 0) == rows_qkv * cfg.hidden * 2 // 16384
    err = mk.mk_host_plan_simulate(cfg, opts, 148, steps=1, seed=7, timeout_ms=20000)
    assert err == ""


def test_use_tcgen05_option():
    """use_tcgen05: automatic (tensor-core tiles at batch > 1), forced off
    (CUDA-core pages at any batch), forced on (refused at batch 1, where every
    product is a matrix-vector product); the tensor-core QKV / O needs it on."""
    cfg = cfg_for("llama1b_b16", max_batch=16)
    F = cfg.ffn
    auto, *_ = mk.mk_host_plan(cfg, mk.plan_opts(batch=16), 148)
    on, *_ = mk.mk_host_plan(cfg, mk.plan_opts(batch=16, use_tcgen05=1), 148)
    off, *_ = mk.mk_host_plan(cfg, mk.plan_opts(batch=16, use_tcgen05=-1), 148)
    gu_units = lambda ins: sum(i.b for i in ins if i.op == OP["gateup"] and i.layer == 0)
    assert gu_units(auto) == gu_units(on) == F // 64          # 128-row tiles of 64 gate + 64 up rows
    rows_per_page = 16384 // (2 * cfg.hidden)
    assert gu_units(off) == F // (rows_per_page // 2)           # one page of R/2 gate + R/2 up rows each
    # down K pieces: 1024 columns on the tensor cores, 2048 (the page rows' width) on CUDA cores
    pieces = lambda ins: sorted({i.c for i in ins if i.op == OP["down"] and i.layer == 0})
    assert pieces(on) == list(range(F // 1024)) and pieces(off) == list(range(F // 2048))
    assert mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=16, use_tcgen05=-1), 148, steps=1, seed=3,
                                    timeout_ms=20000) == ""
    cfg1 = cfg_for("llama1b")
    for bad in (mk.plan_opts(batch=1, use_tcgen05=1), mk.plan_opts(batch=16, use_tcgen05=2),
                mk.plan_opts(batch=16, use_tcgen05=-1, tensor_qkv_o=True)):
        with pytest.raises(mk.MkError) as e:
            mk.mk_host_plan(cfg1 if bad.batch == 1 else cfg, bad, 148)
        assert e.value.code == mk.MK_ERR_INVALID_ARG
    # off at batch 1 is the batch-1 default
    a, *_ = mk.mk_host_plan(cfg1, mk.plan_opts(batch=1), 148)
    b, *_ = mk.mk_host_plan(cfg1, mk.plan_opts(batch=1, use_tcgen05=-1), 148)
    assert [bytes(x) for x in a] == [bytes(x) for x in b]


@pytest.mark.parametrize("tqo", [False, True])
@pytest.mark.parametrize("sched,num_ctas", [("static", 37), ("dynamic", 148), ("dynamic", 16), ("event", 148),
                                            ("event", 16)])
def test_batched_plan_other_grids(tqo, sched, num_ctas):
    """Batched plans on smaller grids and with the dynamic queue: every
    matrix row of every layer is covered exactly once, and the host
    simulation of the counter protocol completes."""
    cfg = cfg_for("llama1b_b16", max_batch=16)
    opts = mk.plan_opts(batch=16, sched=sched, tensor_qkv_o=tqo)
    instrs, off, ln, info = mk.mk_host_plan(cfg, opts, num_ctas)
    assert [i.seq for i in sorted(instrs, key=lambda i: i.seq)] == list(range(len(instrs)))
    H, F = cfg.hidden, cfg.ffn
    qkv_rows = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
    rows_per_unit = {"qkv": 128 if tqo else 8192 // H, "oproj": 128 if tqo else 8192 // (cfg.n_q_heads * cfg.head_dim),
                     "gateup": 64}
    total = {"qkv": qkv_rows, "oproj": H, "gateup": F}
    for l in (0, cfg.n_layers // 2, cfg.n_layers - 1):
        for op, n in total.items():
            units = sorted(u for i in instrs if i.op == OP[op] and i.layer == l for u in range(i.a, i.a + i.b))
            assert units == list(range(n // rows_per_unit[op])), (op, l)
        for k in range(F // 2048):
            units = sorted(u for i in instrs if i.op == OP["down"] and i.layer == l and i.c == k
                           for u in range(i.a, i.a + i.b))
            assert units == list(range(H // 128)), ("down", l, k)
    err = mk.mk_host_plan_simulate(cfg, opts, num_ctas, steps=1, seed=11, timeout_ms=30000)
    assert err == ""


def _shape_grid():
    """Shapes the engine accepts, beyond the named workloads: every hidden
    size, both head dims, several GQA groups, FFN widths around the K-piece
    size and vocabularies that leave a partial LM-head page."""
    import random
    rng = random.Random(17)
    out = []
    for H in (256, 512, 1024, 2048, 4096):
        for d in (64, 128):
            for qd in (256, 1024, 4096):
                nq = qd // d
                for g in (1, 2, 4, 8):
                    if nq % g or (8192 // H) > d or d % (8192 // H):
                        continue
                    F = rng.choice([256, 512, 1024, 2048, 6144, 14336, 16384])
                    if F % max(1, (8192 // H) // 2):
                        continue
                    V = rng.choice([1000, 4096, 32003])
                    out.append((H, d, nq, nq // g, F, V))
    rng.shuffle(out)
    return out[:24]


@pytest.mark.parametrize("H,d,nq,nkv,F,V", _shape_grid())
def test_plan_structure_shape_grid(H, d, nq, nkv, F, V):
    """Page coverage, queue order and counter targets for shapes beyond the
    named workloads, on a full and a small grid, and the counter protocol on
    the small grid."""
    shape = dict(n_layers=2, hidden=H, n_q_heads=nq, n_kv_heads=nkv, head_dim=d, ffn=F, vocab=V,
                 rms_eps=1e-5, rope_theta=1e4, tied=V == 4096)
    cfg = mk.make_config(shape, 1, 300)
    for num_ctas in (148, 13):
        instrs, off, ln, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=1), num_ctas)
        check_structure(cfg, instrs, off, ln, num_ctas)
    err = mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=1), 13, steps=1, seed=H + F, timeout_ms=30000)
    assert err == ""
    instrs, off, ln, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=1, sched="dynamic"), 13)
    check_structure(cfg, instrs, off, ln, 13, dynamic=True)
    err = mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=1, sched="dynamic"), 13, steps=2, seed=V,
                                   timeout_ms=30000)
    assert err == ""
    err = mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=1, sched="event"), 13, steps=2, seed=V + 1,
                                   timeout_ms=30000)
    assert err == ""


@pytest.mark.parametrize("F", [768, 1280, 3072, 18432])
def test_unsupported_ffn_widths_rejected(F):
    """FFN widths outside the documented set are refused by the planner."""
    shape = dict(n_layers=2, hidden=1024, n_q_heads=16, n_kv_heads=4, head_dim=64, ffn=F, vocab=4096,
                 rms_eps=1e-5, rope_theta=1e4, tied=True)
    with pytest.raises(mk.MkError) as e:
        mk.mk_host_plan(mk.make_config(shape, 1, 64), mk.plan_opts(batch=1), 8)
    assert e.value.code == mk.MK_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("seed", [101, 202, 303])
@pytest.mark.parametrize("name,batch,kw", [("llama1b", 1, {}), ("llama1b", 1, {"sched": "dynamic"}),
                                            ("llama1b", 1, {"sched": "event"}), ("llama1b_b16", 16, {"sched": "event"}),
                                            ("llama8b", 1, {}), ("llama1b_b16", 16, {}),
                                            ("llama1b_b16", 16, {"tensor_qkv_o": True})])
def test_simulation_more_seeds(seed, name, batch, kw):
    """The counter protocol under other random delay patterns, on the full
    grid, for the benchmarked plans (two steps, so the epoch targets of a
    second step are exercised too)."""
    cfg = cfg_for(name, max_batch=batch)
    err = mk.mk_host_plan_simulate(cfg, mk.plan_opts(batch=batch, **kw), 148, steps=2, seed=seed, timeout_ms=60000)
    assert err == ""
