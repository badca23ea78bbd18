#!/usr/bin/env python
"""Decode-step benchmark of the megakernel engine.

A step is one autoregressive decode step (every instruction class of the
decode path: RMSNorm + QKV + RoPE + KV append, split-KV GQA attention,
O projection, RMSNorm + gate/up + SiLU, down projection, final norm + LM head +
argmax) of the Llama-3.2-1B-shaped model at batch 1, KV cache pre-filled to
1024 positions, on seeded synthetic weights (bf16 ~N(0, 0.02)).  Prints one
JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mk|reference]

N > 1 runs under torchrun: batch-1 decode does not shard, so every rank runs
an independent replica ("replicas only", weak scaling); value = all ranks'
steps / max time.  The batched workload (16 independent sequences) is split
data-parallel: rank r decodes its own contiguous slice of the sequences, with
the weights replicated and no collective (strong scaling); value = whole-batch
steps / max time.
--impl reference times the CPU oracle (the only reference this build has).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode steps/sec & µs/step (Llama-1B shape, batch 1); HBM GB/s as % of roofline"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=128)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--workload", default="llama1b")
    ap.add_argument("--exec-mode", default="megakernel",
                    choices=["megakernel", "megakernel_generic", "per_op", "per_op_graph"])
    ap.add_argument("--sched", default="static", choices=["static", "dynamic", "event"])
    ap.add_argument("--kv-splits", type=int, default=0)
    ap.add_argument("--l2-prefetch-kb", type=int, default=0)
    ap.add_argument("--inflight", type=int, default=0, help="bulk-copy pages in flight per CTA (0 = default)")
    ap.add_argument("--tensor-qkv-o", action="store_true",
                    help="batched plans: QKV and O projection on the tensor cores too")
    ap.add_argument("--use-tcgen05", type=int, default=0, choices=[-1, 0, 1],
                    help="batched plans: tensor cores for the matrix instructions (0 = automatic, -1 = off)")
    ap.add_argument("--no-compare-modes", action="store_true",
                    help="skip timing the per-op path (with and without a CUDA graph) and the dynamic queue on "
                         "the same workload after the timed region (single GPU; reported under \"comparison\")")
    ap.add_argument("--compare-steps", type=int, default=32, help="timed steps of each comparison path")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true",
                    help="skip the traced step (per-instruction-class time breakdown) after the timed region")
    ap.add_argument("--no-logits", action="store_true", help="do not write logits_out")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: truncate the model to this many layers (not a bench number)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def src_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "decode_megakernel_interpreter_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("src_hash") == src_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while running."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index: int):
        self.samples = []
        self.reasons = set()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:
                import torch
                pr = torch.cuda.get_device_properties(index)
                bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            pass
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                f = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = f(self.h)
                for n, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(n)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def step_bytes(shape, weight_bytes: int, positions, logits: bool) -> float:
    """Algorithmic HBM bytes of one step, averaged over the timed steps:
    weights streamed once for all sequences (+ norm vectors), and per sequence
    one embedding row, the KV cache read over positions 0..pos, the new K/V
    row written and fp32 logits written.  positions[i][b]: position of
    sequence b at step i."""
    L, H, d, nkv = shape.n_layers, shape.hidden, shape.head_dim, shape.n_kv_heads
    norms = (2 * L + 1) * H * 2
    per_pos = L * nkv * d * 2 * 2
    tot = 0.0
    for row in positions:
        tot += weight_bytes + norms
        for p in row:
            tot += H * 2 + per_pos * (p + 1) + per_pos + (shape.vocab * 4 if logits else 0)
    return tot / len(positions)


def max_over_ranks(ms: float, pg, device: str) -> float:
    """The job's time: the slowest rank's (every rank takes part; `pg` is
    torch.distributed or None for a single process)."""
    if pg is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, steps: int, ms: float) -> float:
    """Whole-job throughput of independent replicas: every rank's steps over
    the job's time."""
    return world * steps / (ms / 1e3)


def shard_sequences(batch: int, world: int, rank: int):
    """Data-parallel split of a batch of independent sequences: rank r decodes
    the contiguous slice [start, start + count); slices differ by at most one
    sequence and cover the batch once."""
    if world > batch:
        raise SystemExit(f"{world} ranks for {batch} sequences: every rank needs at least one")
    base, rem = divmod(batch, world)
    start = rank * base + min(rank, rem)
    return start, base + (1 if rank < rem else 0)


def sharded_rate(steps: int, ms: float) -> float:
    """Whole-job throughput of a batch split across ranks: every rank advances
    its slice by `steps` tokens, so the job advances the whole batch `steps`
    times in the slowest rank's time."""
    return steps / (ms / 1e3)


def dist_setup(n):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if n > 1 and world != n:
        raise SystemExit(f"--gpus {n} needs torchrun with {n} ranks (WORLD_SIZE={world})")
    return world, rank, local


def workload_config(w) -> dict:
    """The config keys both arms report for a workload."""
    s = w.shape
    lengths = [int(x) for x in w.lengths()]
    family = {4096: "Llama-3.1-8B", 2048: "Llama-3.2-1B"}.get(s.hidden)
    desc = w.name
    if family:
        desc += (f": {family} shape ({s.n_layers} layers, hidden {s.hidden}, {s.n_q_heads}/{s.n_kv_heads} heads, "
                 f"head_dim {s.head_dim}, ffn {s.ffn}, vocab {s.vocab}, {'tied' if s.tied else 'untied'})")
    if w.ragged is None:
        ctx = lengths[0]
        desc += f", batch {w.batch}, KV pre-filled to {ctx}"
    else:
        ctx = f"U[{w.ragged[0]}, {w.ragged[1]}] per sequence (mean {sum(lengths) / len(lengths):.0f})"
        desc += f", batch {w.batch}, KV pre-filled to {ctx}"
    return {"workload": desc, "batch": w.batch, "context": ctx}


def _omp():
    """The OpenMP runtime the oracle library links (None if not loadable)."""
    import ctypes
    try:
        return ctypes.CDLL("libgomp.so.1")
    except OSError:
        return None


def host_cores() -> int:
    """Threads the OpenMP oracle runs with on this host."""
    g = _omp()
    if g is not None:
        return int(g.omp_get_max_threads())
    if os.environ.get("OMP_NUM_THREADS"):
        return int(os.environ["OMP_NUM_THREADS"])
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_steps(w, model, steps: int, warmup: int, budget_s: float):
    """Greedy decode steps of the whole batch (every sequence at its own
    context length) with the fp64 oracle: `warmup` untimed steps, then up to
    `steps` timed ones, stopping early once `budget_s` seconds are spent.
    Returns (timed steps, seconds, warm-up steps done)."""
    import numpy as np
    import oracle
    import synth
    s = w.shape
    lengths = [int(x) for x in w.lengths()]
    k, v = synth.alloc_kv(s, w.batch, max(lengths) + steps + warmup + 2)
    synth.fill_kv_prefix(s, k, v, lengths)
    orc = oracle.Oracle(s, model, "f64")
    tok = [int(t) for t in synth.first_tokens(w)]
    pos = list(lengths)

    def step():
        for b in range(w.batch):
            lg = orc.decode_step(k, v, b, tok[b], pos[b])
            tok[b], pos[b] = int(np.argmax(lg)), pos[b] + 1

    t0 = time.perf_counter()
    done_w = 0
    for _ in range(warmup):  # untimed, bounded like the timed part
        step()
        done_w += 1
        if time.perf_counter() - t0 > budget_s / 2:
            break
    n, t0 = 0, time.perf_counter()
    while n < steps:
        step()
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return n, time.perf_counter() - t0, done_w


def run_reference(args, world, rank):
    """The CPU oracle (fp64) on this host's cores: the workload's decode steps
    (all of its sequences), a bounded sample of them."""
    if rank != 0:
        return
    import synth
    w = synth.WORKLOADS[args.workload]
    model = synth.make_model(w.shape)
    n, el, done_w = oracle_steps(w, model, args.steps, args.warmup, budget_s=150.0)
    val = n / el
    sample = (f"{n} of the {args.steps} requested decode steps of {args.workload} "
              f"({w.batch} sequence{'s' if w.batch > 1 else ''} each; {done_w} untimed warm-up), fp64 oracle")
    out = {"metric": METRIC, "value": val, "unit": "steps/s", "n_gpus": world, "steps": n, "warmup": done_w,
           "ms_per_step": 1e3 * el / n, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f64", "data": "synthetic (seeded bf16 weights ~N(0,0.02), KV ~N(0,1))",
           "config": workload_config(w),
           "impl": "reference",
           "cpu_baseline": {"value": val, "unit": "steps/s", "cores": host_cores(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": val, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def cpu_baseline(model, w, seconds=15.0):
    n, el, _ = oracle_steps(w, model, 60, 0, budget_s=seconds)
    out = {"value": n / el, "unit": "steps/s", "cores": host_cores(), "kind": "oracle",
           "sample": f"{n} consecutive decode steps of {w.name} ({w.batch} sequence{'s' if w.batch > 1 else ''} "
                     f"each, at the workload's context lengths), fp64 oracle, {el:.1f} s of host time"}
    g = _omp()
    if g is not None and w.batch == 1:
        # the same oracle on one thread (a batched step would take minutes there)
        prev = g.omp_get_max_threads()
        g.omp_set_num_threads(1)
        try:
            n1, el1, _ = oracle_steps(w, model, 60, 0, budget_s=seconds / 2)
        finally:
            g.omp_set_num_threads(prev)
        out["single_thread"] = {"value": n1 / el1, "unit": "steps/s", "cores": 1,
                                "sample": f"{n1} decode steps of {w.name}, {el1:.1f} s"}
    return out


def breakdown(eng, mk, info, tokens, pos0, logits, nxt):
    import numpy as np
    import torch
    eng.plan(**{**eng.plan_kw, "trace": True})
    eng.decode_step(tokens, pos0, logits, nxt)
    torch.cuda.synchronize()
    tr = eng.trace().astype(np.int64)
    eng.plan(**eng.plan_kw)
    ops = tr[:, 7] & 0xFF
    t_start = tr[:, 0].min()
    total = tr[:, 4].max() - t_start
    out = {"step_us_traced": total / 1e3}
    if os.environ.get("MK_TRACE_DUMP"):
        np.save(os.environ["MK_TRACE_DUMP"], tr)
    for op in sorted(set(ops.tolist())):
        m = ops == op
        wait = (tr[m, 1] - tr[m, 0]) / 1e3
        stage = (tr[m, 2] - tr[m, 1]) / 1e3
        pages = (tr[m, 3] - tr[m, 2]) / 1e3
        sig = (tr[m, 4] - tr[m, 3]) / 1e3
        out[mk.OP_NAMES[int(op)]] = {"count": int(m.sum()), "mean_wait_us": float(wait.mean()),
                                     "mean_stage_us": float(stage.mean()), "mean_pages_us": float(pages.mean()),
                                     "mean_signal_us": float(sig.mean()),
                                     "mean_body_us": float((tr[m, 3] - tr[m, 1]).mean() / 1e3),
                                     "mean_pages_per_instr": float(tr[m, 11].mean()),
                                     "consumer_page_waits": int((tr[m, 8] & 0xffffffff).sum()),
                                     "tagged_load_retries": int((tr[m, 8] >> 32).sum()),
                                     "loader_ring_full": int(tr[m, 9].sum())}
        if (tr[m, 10] > 0).all():  # attention: the page loop and the merges after it
            out[mk.OP_NAMES[int(op)]]["mean_page_loop_us"] = float(((tr[m, 10] - tr[m, 2]) / 1e3).mean())
            out[mk.OP_NAMES[int(op)]]["mean_merge_us"] = float(((tr[m, 3] - tr[m, 10]) / 1e3).mean())
    return out


def main():
    args = parse()
    world, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    import numpy as np
    import torch
    import decode_megakernel_interpreter_b200 as mk
    from decode_megakernel_interpreter_b200 import harness
    import synth

    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        pg = dist
    w = synth.WORKLOADS[args.workload]
    if args.layers:
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}_{args.layers}layers",
                                shape=dataclasses.replace(w.shape, n_layers=args.layers))
    s = w.shape
    K, W = args.steps, args.warmup
    all_lengths = [int(x) for x in w.lengths()]
    all_first = [int(x) for x in synth.first_tokens(w)]
    # batched workloads: this rank's slice of the sequences (data parallel);
    # batch-1 workloads: a full replica per rank
    sharded = w.batch > 1 and world > 1
    seq0, B = shard_sequences(w.batch, world, rank) if sharded else (0, w.batch)
    lengths = all_lengths[seq0:seq0 + B]
    max_seq = max(lengths) + K + W + 2
    model = synth.make_model(s)
    dev = harness.upload_model(model, s.tied)
    k, v = synth.alloc_kv(s, B, max_seq)
    synth.fill_kv_prefix(s, k, v, lengths)
    kc, vc = harness.upload_kv(k, v)
    del k, v
    eng = harness.make_engine(s, dev, kc, vc, B, max_seq)
    plan_kw = dict(batch=B, kv_splits=args.kv_splits, sched=args.sched, exec_mode=args.exec_mode,
                   l2_prefetch_kb=args.l2_prefetch_kb, max_inflight_pages=args.inflight,
                   tensor_qkv_o=args.tensor_qkv_o, use_tcgen05=args.use_tcgen05 if B > 1 else 0)
    eng.plan_kw = plan_kw
    info = eng.plan(**plan_kw)
    stream = torch.cuda.current_stream()
    first = torch.tensor(all_first[seq0:seq0 + B], dtype=torch.int32, device="cuda")
    tokens = first.clone()  # next_tokens_out aliases tokens: device-to-device feedback
    # positions of every sequence at every step (row i: step i)
    pos_host = torch.tensor([[n + i for n in lengths] for i in range(max(K, W) + 1)], dtype=torch.int32)
    pos_all = pos_host.to("cuda")
    logits = None if args.no_logits else torch.empty(B, s.vocab, dtype=torch.float32, device="cuda")
    lptr = logits.data_ptr() if logits is not None else None

    def step(i):
        rc = mk.mk_decode_step(eng.h, tokens.data_ptr(), pos_all[i].data_ptr(), lptr, tokens.data_ptr(),
                               stream.cuda_stream)
        if rc != mk.MK_OK:
            raise mk.MkError(rc, "mk_decode_step")

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    rc = eng.status()
    if rc != mk.MK_OK:
        raise mk.MkError(rc, "warm-up")
    tokens.copy_(first)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev0.record(stream)
        for i in range(K):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    ms = ev0.elapsed_time(ev1)
    rc = eng.status()
    if rc != mk.MK_OK:
        raise mk.MkError(rc, "timed steps")
    ms = max_over_ranks(ms, pg, "cuda")
    us_step = 1e3 * ms / K
    value = sharded_rate(K, ms) if sharded else job_rate(world, K, ms)
    launches_per_step = 1 if args.exec_mode.startswith("megakernel") else s.n_layers * 5 + 1

    # the comparison paths on the same workload and buffers (opt-in): re-plan,
    # warm up, time K steps the same way, then restore the measured plan
    comparison = None
    if not args.no_compare_modes and world == 1:
        comparison = {"megakernel": {"us_per_step": us_step, "plan": {"exec_mode": args.exec_mode,
                                                                       "sched": args.sched}}}
        Kc = max(1, min(K, args.compare_steps))
        for label, over in (("per_op", dict(exec_mode="per_op")), ("per_op_graph", dict(exec_mode="per_op_graph")),
                            ("dynamic_queue", dict(sched="dynamic", exec_mode="megakernel")),
                            ("event_queue", dict(sched="event", exec_mode="megakernel"))):
            kw = {**plan_kw, **over}
            if kw == plan_kw:
                continue
            eng.plan(**kw)
            tokens.copy_(first)
            for i in range(W):
                step(i)
            torch.cuda.synchronize()
            tokens.copy_(first)
            c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            c0.record(stream)
            for i in range(Kc):
                step(i)
            c1.record(stream)
            torch.cuda.synchronize()
            rc = eng.status()
            if rc != mk.MK_OK:
                raise mk.MkError(rc, f"comparison {label}")
            comparison[label] = {"us_per_step": 1e3 * c0.elapsed_time(c1) / Kc, "steps": Kc, "plan": over}
        info = eng.plan(**plan_kw)
        tokens.copy_(first)

    # end to end through the C ABI with host buffers: per step copy the token
    # and position in from pinned memory, run, read the next token back
    e2e = None
    if not args.no_e2e:
        h_tok = torch.empty(B, dtype=torch.int32, pin_memory=True)
        h_pos = torch.empty(B, dtype=torch.int32, pin_memory=True)
        h_next = torch.empty(B, dtype=torch.int32, pin_memory=True)
        d_tok = torch.empty(B, dtype=torch.int32, device="cuda")
        d_pos = torch.empty(B, dtype=torch.int32, device="cuda")
        d_next = torch.empty(B, dtype=torch.int32, device="cuda")
        h_tok.copy_(first.cpu())
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(K):
            h_pos.copy_(pos_host[i])
            d_tok.copy_(h_tok, non_blocking=True)
            d_pos.copy_(h_pos, non_blocking=True)
            rc = mk.mk_decode_step(eng.h, d_tok.data_ptr(), d_pos.data_ptr(), lptr, d_next.data_ptr(),
                                   stream.cuda_stream)
            if rc != mk.MK_OK:
                raise mk.MkError(rc, "e2e step")
            h_next.copy_(d_next, non_blocking=True)
            stream.synchronize()
            h_tok.copy_(h_next)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1)
        ems = max_over_ranks(ems, pg, "cuda")
        e2e = {"value": sharded_rate(K, ems) if sharded else job_rate(world, K, ems), "unit": "steps/s",
               "h2d_bytes_per_step": 8 * B,
               "d2h_bytes_per_step": 4 * B, "us_per_step": 1e3 * ems / K}

    bd = None
    if not args.no_breakdown:
        bd = breakdown(eng, mk, info, tokens, pos_all[0], logits, torch.empty_like(tokens))
    eng.close()

    if rank == 0:
        peak, peak_kind = peaks()
        positions = [[n + i for n in lengths] for i in range(K)]
        bytes_step = step_bytes(s, info.weight_bytes_per_step, positions, logits is not None)
        achieved = bytes_step / (us_step * 1e-6) / 1e9
        out = {
            "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": us_step / 1e3, "us_per_step": us_step, "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": "f32", "operand_dtype": "bf16 weights and KV cache",
            "exchange": ("fp32 rounded to 22 significant bits with a 2-bit step tag in the low mantissa bits"
                         + ("; tensor-core operands bf16 hi + lo (about 16 significant bits)"
                            if B > 1 and args.use_tcgen05 >= 0 else "")),
            "data": "synthetic",
            "config": {**workload_config(w), "exec_mode": args.exec_mode, "sched": args.sched,
                       "kv_splits": info.kv_splits, "ctas": info.num_ctas, "smem_pages": info.num_pages,
                       "interpreter": "shape-specialised" if info.kernel_variant == 1 else "shape-generic",
                       "parallelism": ("data parallel: sequences split across ranks, weights replicated, "
                                       "no collective" if sharded else
                                       "replicas only" if world > 1 else "single GPU"),
                       **({"sequences_per_rank": B} if sharded else {}),
                       "l2": f"inputs larger than L2 (weights streamed once per step, "
                             f"{info.weight_bytes_per_step / 1e9:.2f} GB; L2 126 MB)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_kind": peak_kind, "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                         "traffic": ncu_traffic(args.workload), "algorithmic_bytes_per_step": bytes_step,
                         "kernel": "mk::interp_kernel"},
            "clocks": clk.summary(),
            "gpu_launches": K * launches_per_step,
        }
        if e2e:
            out["e2e"] = e2e
        if bd:
            out["breakdown"] = bd
        if comparison is not None:
            out["comparison"] = comparison
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(model, w)
        print(json.dumps(out), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
