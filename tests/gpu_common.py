"""Shared helpers of the GPU parity tests (seeded workloads, oracle
comparisons).  Imported by tests only."""
from __future__ import annotations

import numpy as np

import oracle
import synth

ATOL, RTOL = 2e-2, 1e-2  # logit tolerance: |gpu - oracle| <= ATOL + RTOL * |oracle|
U32 = 2.0 ** -24         # unit roundoff of fp32 (the engine's accumulation type)
NORM_SIGMA = 0.3         # spread of the seeded norm weights of the gamma tests


def bf16_ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def bf16_ulp(bits: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at each value (8 significant bits)."""
    e = ((bits.astype(np.int32) >> 7) & 0xFF)
    return np.ldexp(1.0, np.maximum(e, 1) - 127 - 7)


def gamma_n(n: int) -> float:
    """Higham's gamma_n = n u / (1 - n u): a dot product of length n summed in
    fp32 in any order is within gamma_n * sum |w_j x_j| of the exact value."""
    return n * U32 / (1.0 - n * U32)


def abs_kv_weights(model: dict, layer: int):
    """|W_k|, |W_v| of one layer as float32 (the bound's magnitudes)."""
    L = model["layers"][layer]
    return (np.abs(synth.bf16_bits_to_f32(L["wk"])), np.abs(synth.bf16_bits_to_f32(L["wv"])))


def kv_row_bounds(model: dict, shape, layer: int, x_in: np.ndarray, absw=None):
    """Per-element error bounds (K, V) of one layer's K/V row before its bf16
    rounding.  a = rms(x_in) * gamma (the oracle's exact input of the layer);
    each element is a dot product of length H, so its fp32 value is within
    gamma_H * sum_j |W_ij| |a_j| (the bound the oracle's own matvec pin uses);
    (layer + 2) such terms cover, to first order, this dot product, the
    RMSNorm staging and the residual stream's error inherited from the earlier
    layers.  RoPE mixes the pair (i, i + d/2) with |cos|, |sin| <= 1, so a K
    element's bound is the sum of its pair's."""
    H, d = shape.hidden, shape.head_dim
    L = model["layers"][layer]
    g = synth.bf16_bits_to_f32(L["attn_norm"]).astype(np.float64)
    x = x_in.astype(np.float64)
    a = np.abs(x / np.sqrt(np.mean(x * x) + shape.rms_eps) * g).astype(np.float32)
    c = (layer + 2) * gamma_n(H)
    wk, wv = absw if absw is not None else abs_kv_weights(model, layer)
    ek = c * (wk @ a).astype(np.float64)
    ev = c * (wv @ a).astype(np.float64)
    ek = ek.reshape(-1, d)
    ek = ek + np.concatenate([ek[:, d // 2:], ek[:, :d // 2]], axis=1)
    return ek.reshape(shape.n_kv_heads, d), ev.reshape(shape.n_kv_heads, d)


def kv_row_mismatch(gpu_bits: np.ndarray, ora_bits: np.ndarray, bound: np.ndarray) -> str:
    """'' when every element of the GPU's bf16 row is within one bf16 ulp plus
    `bound` (the fp32 error bound of the value before rounding) of the
    oracle's.  Rounding both sides' values to bf16 can differ by at most
    their distance plus one ulp.  Else a message naming the worst element."""
    g = synth.bf16_bits_to_f32(gpu_bits).astype(np.float64)
    o = synth.bf16_bits_to_f32(ora_bits).astype(np.float64)
    slack = bf16_ulp(ora_bits) + bound
    bad = np.abs(g - o) > slack
    if not bad.any():
        return ""
    i = np.unravel_index(np.argmax(np.where(bad, np.abs(g - o) / slack, -1)), g.shape)
    ulps = np.abs(bf16_ordered(gpu_bits) - bf16_ordered(ora_bits))
    return (f"{int(bad.sum())} elements off; worst at {i}: gpu {g[i]!r} oracle {o[i]!r} "
            f"({int(ulps[i])} ulp, bound {bound[i]:.3g})")


def layer_inputs(model: dict, token: int, dump: dict) -> list:
    """x_in of every layer from an oracle dump: the embedding row, then each
    layer's output residual."""
    emb = synth.bf16_bits_to_f32(model["embed"][token]).astype(np.float64)
    return [emb] + [dump["x_out"][l] for l in range(dump["x_out"].shape[0] - 1)]


class HostSetup:
    """Host model + the oracle's own KV cache for one workload."""

    def __init__(self, shape: synth.ModelShape, batch: int, max_seq: int, model=None):
        self.shape = shape
        self.batch = batch
        self.max_seq = max_seq
        self.model = model if model is not None else synth.make_model(shape)
        self.k, self.v = synth.alloc_kv(shape, batch, max_seq)
        self.orc = oracle.Oracle(shape, self.model, "f64")
        self._absw = {}

    def fill_prefix(self, lengths):
        synth.fill_kv_prefix(self.shape, self.k, self.v, lengths)

    def prefill_prompt(self, tokens, b=0) -> np.ndarray:
        return self.orc.prefill(self.k, self.v, b, tokens)

    def decode(self, b: int, token: int, pos: int):
        """Oracle logits of one step and the K/V error bounds of every layer
        ([L][n_kv][d] each)."""
        logits, dump = self.orc.decode_step(self.k, self.v, b, token, pos, dump=True)
        xs = layer_inputs(self.model, token, dump)
        bk, bv = [], []
        for l in range(self.shape.n_layers):
            if l not in self._absw:
                self._absw[l] = abs_kv_weights(self.model, l)
            k_, v_ = kv_row_bounds(self.model, self.shape, l, xs[l], self._absw[l])
            bk.append(k_)
            bv.append(v_)
        return logits, np.stack(bk), np.stack(bv)


class StepCheck:
    """Per-step logit and greedy-id comparison against the oracle.

    eps = the step's largest |gpu - oracle| logit difference.  If the oracle's
    top-2 margin exceeds 2 eps, the GPU's argmax can only be the oracle's
    (top1 - eps > second + eps), so the ids must be identical; inside that
    margin (a near tie) any id whose oracle logit is within 2 eps of the
    maximum is a correct greedy pick.  Counts are kept for the parity log."""

    def __init__(self):
        self.steps = 0
        self.near_ties = 0
        self.id_mismatches = 0
        self.max_abs = 0.0
        self.max_rel = 0.0

    def check(self, gpu_logits: np.ndarray, ora_logits: np.ndarray, gpu_next: int, what: str):
        g = gpu_logits.astype(np.float64)
        diff = np.abs(g - ora_logits)
        eps = float(diff.max())
        self.steps += 1
        self.max_abs = max(self.max_abs, eps)
        self.max_rel = max(self.max_rel, float(np.max(diff / np.maximum(np.abs(ora_logits), 1e-3))))
        bad = diff > ATOL + RTOL * np.abs(ora_logits)
        assert not bad.any(), f"{what}: {int(bad.sum())} logits outside atol 2e-2 / rtol 1e-2 (max abs {eps})"
        top = int(np.argmax(ora_logits))
        top2 = np.partition(ora_logits, -2)[-2:]
        margin = float(top2[1] - top2[0])
        if gpu_next != top:
            self.id_mismatches += 1
        if margin > 2 * eps:
            assert gpu_next == top, f"{what}: greedy id {gpu_next} != oracle {top} (margin {margin:.3g}, eps {eps:.3g})"
        else:
            self.near_ties += 1
            assert ora_logits[gpu_next] >= ora_logits[top] - 2 * eps, f"{what}: greedy id outside the tie band"

    def record(self) -> dict:
        return {"steps": self.steps, "near_ties": self.near_ties, "id_mismatches": self.id_mismatches,
                "max_abs": self.max_abs, "max_rel": self.max_rel}
