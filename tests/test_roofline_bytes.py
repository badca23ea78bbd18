"""The roofline numerator: the algorithmic bytes of a step that bench.py
divides by the measured time, pinned to the model's parameter count and the
KV-cache geometry (closed forms, no GPU)."""
import importlib.util
import os

import pytest

import decode_megakernel_interpreter_b200 as mk
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_bytes_under_test", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_parameter_counts():
    # Llama-3.2-1B (tied head) and Llama-3.1-8B (untied) totals
    assert synth.LLAMA_1B.n_params() == 1_235_814_400
    assert synth.LLAMA_8B.n_params() == 8_030_261_248


@pytest.mark.parametrize("name", ["llama1b", "llama8b"])
def test_streamed_weights_are_every_parameter_once(name):
    """Plan weight bytes + norm vectors + one embedding row = every bf16
    parameter read once (a tied head is the embedding table, read once as the
    LM head; an untied model reads one embedding row, not the table)."""
    w = synth.WORKLOADS[name]
    s = w.shape
    cfg = mk.make_config(s, 1, w.context + w.steps)
    *_, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=1), 148)
    norms = (2 * s.n_layers + 1) * s.hidden * 2
    streamed = info.weight_bytes_per_step + norms + 2 * s.hidden
    params = s.n_params() - (0 if s.tied else s.vocab * s.hidden)
    assert streamed == 2 * params + 2 * s.hidden


def test_llama1b_step_bytes_closed_form():
    """Context 1024, 128 greedy steps: weights once, K/V read over positions
    0..p and the new row written (32 KiB per position), fp32 logits."""
    b = _bench()
    w = synth.WORKLOADS["llama1b"]
    s = w.shape
    cfg = mk.make_config(s, 1, w.context + w.steps)
    *_, info = mk.mk_host_plan(cfg, mk.plan_opts(batch=1), 148)
    positions = [[w.context + i] for i in range(w.steps)]
    got = b.step_bytes(s, info.weight_bytes_per_step, positions, True)
    per_pos = s.n_layers * s.n_kv_heads * s.head_dim * 2 * 2
    assert per_pos == 32_768
    mean_rows = sum(p + 2 for (p,) in positions) / len(positions)  # 0..p read, row p written
    want = (2 * s.n_params() + 2 * s.hidden) + per_pos * mean_rows + 4 * s.vocab
    assert got == pytest.approx(want, rel=0, abs=1e-3)
    assert round(got) == 2_507_846_656


def test_batched_step_bytes_count_every_sequence():
    """Batch 16: the weights once per step, the K/V of every sequence over its
    own positions, one embedding row and one row of logits per sequence."""
    b = _bench()
    w = synth.WORKLOADS["llama1b_b16"]
    s = w.shape
    cfg = mk.make_config(s, 16, w.max_seq())
    *_, info16 = mk.mk_host_plan(cfg, mk.plan_opts(batch=16), 148)
    *_, info1 = mk.mk_host_plan(mk.make_config(s, 1, 2048), mk.plan_opts(batch=1), 148)
    assert info16.weight_bytes_per_step == info1.weight_bytes_per_step
    lengths = [int(x) for x in w.lengths()]
    positions = [[n + i for n in lengths] for i in range(3)]
    got = b.step_bytes(s, info16.weight_bytes_per_step, positions, True)
    per_pos = s.n_layers * s.n_kv_heads * s.head_dim * 2 * 2
    norms = (2 * s.n_layers + 1) * s.hidden * 2
    kv = sum(per_pos * (p + 2) for row in positions for p in row) / len(positions)
    want = info16.weight_bytes_per_step + norms + 16 * (2 * s.hidden + 4 * s.vocab) + kv
    assert got == pytest.approx(want, rel=0, abs=1e-3)
