"""Shared helpers of the GPU parity tests (seeded workloads, oracle
comparisons).  Imported by tests only."""
from __future__ import annotations

import numpy as np

import oracle
import synth

ATOL, RTOL = 2e-2, 1e-2  # logit tolerance: |gpu - oracle| <= ATOL + RTOL * |oracle|


def bf16_ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def kv_row_mismatch(gpu_bits: np.ndarray, ora_bits: np.ndarray, rel_floor: float = 1e-4) -> str:
    """'' when every element of the GPU's bf16 rows is within one bf16 ulp of
    the oracle's, or within rel_floor * max|oracle| of it: an element that
    is small through cancellation has a bf16 ulp far below the fp32 error of
    the value being rounded (which scales with the row's magnitude and the
    depth of the layer), so there the two sides cannot take the same rounding
    decision.  Else a message naming the worst element."""
    ulps = np.abs(bf16_ordered(gpu_bits) - bf16_ordered(ora_bits))
    g = synth.bf16_bits_to_f32(gpu_bits).astype(np.float64)
    o = synth.bf16_bits_to_f32(ora_bits).astype(np.float64)
    abs_floor = rel_floor * float(np.abs(o).max())
    bad = (ulps > 1) & (np.abs(g - o) > abs_floor)
    if not bad.any():
        return ""
    i = np.unravel_index(np.argmax(np.where(bad, np.abs(g - o), -1)), g.shape)
    return f"{int(bad.sum())} elements off; worst at {i}: gpu {g[i]!r} oracle {o[i]!r} ({int(ulps[i])} ulp)"


class HostSetup:
    """Host model + the oracle's own KV cache for one workload."""

    def __init__(self, shape: synth.ModelShape, batch: int, max_seq: int, model=None):
        self.shape = shape
        self.batch = batch
        self.max_seq = max_seq
        self.model = model if model is not None else synth.make_model(shape)
        self.k, self.v = synth.alloc_kv(shape, batch, max_seq)
        self.orc = oracle.Oracle(shape, self.model, "f64")

    def fill_prefix(self, lengths):
        synth.fill_kv_prefix(self.shape, self.k, self.v, lengths)

    def prefill_prompt(self, tokens, b=0) -> np.ndarray:
        return self.orc.prefill(self.k, self.v, b, tokens)


def compare_step(gpu_logits: np.ndarray, ora_logits: np.ndarray, gpu_next: int):
    """Returns (ok_logits, near_tie, max_abs, max_rel); asserts nothing."""
    diff = np.abs(gpu_logits.astype(np.float64) - ora_logits)
    ok = bool(np.all(diff <= ATOL + RTOL * np.abs(ora_logits)))
    top2 = np.partition(ora_logits, -2)[-2:]
    margin = float(top2[1] - top2[0])
    near_tie = margin <= 2 * (ATOL + RTOL * abs(float(top2[1])))
    max_rel = float(np.max(diff / np.maximum(np.abs(ora_logits), 1e-3)))
    return ok, near_tie, float(diff.max()), max_rel
