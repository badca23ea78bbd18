"""Seeded synthetic inputs for the decode workloads (shared by the oracle's
tests, the GPU tests and the bench).

Nothing here computes any part of the decode step: it only produces bytes
(bf16 weights, a bf16 KV-cache prefix, token ids, context lengths) from a
counter-based generator defined in ``synth.c``.  The workloads are the ones
the megakernel pages measure (a Llama-3.2-1B-shaped decoder at batch 1,
single sequence) plus a tiny model, a long-context, a batched and an 8B-shaped
variant.  Trained weights are not needed: the shapes and the value
distributions stand in for them (weights ~N(0, 0.02) in bf16, norm weights
1.0, KV cache ~N(0, 1), token ids uniform over the vocabulary).  Parity tests
may also ask for norm weights ~N(1, sigma), one seeded stream per norm vector
(``make_model(..., norm_sigma=...)``), so that a wrong use of them shows.

Seeds: weights 0, KV cache 1, token ids 2, context lengths 3.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field, asdict

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

SEED_WEIGHTS, SEED_KV, SEED_TOKENS, SEED_LENGTHS = 0, 1, 2, 3
WEIGHT_SIGMA = 0.02
KV_SIGMA = 1.0

# tensor-kind ids used in stream keys
K_EMBED, K_LM_HEAD, K_WQ, K_WK, K_WV, K_WO, K_WGATE, K_WUP, K_WDOWN = range(9)
K_ATTN_NORM, K_FFN_NORM, K_FINAL_NORM = 9, 10, 11


def build(force: bool = False) -> str:
    """Compile libsynth.so next to this file (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        u64, i32, vp, dbl, f32 = ctypes.c_uint64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_double, ctypes.c_float
        _lib.syn_key.restype = u64
        _lib.syn_key.argtypes = [u64, u64, u64, u64]
        _lib.syn_normal_bf16.argtypes = [vp, u64, u64, dbl, u64]
        _lib.syn_normal_bf16_mean.argtypes = [vp, u64, u64, dbl, dbl, u64]
        _lib.syn_normal_f32.argtypes = [vp, u64, u64, dbl]
        _lib.syn_uniform_i32.argtypes = [vp, u64, u64, i32, i32]
        _lib.syn_fill_bf16.argtypes = [vp, u64, f32]
    return _lib


def key(seed: int, a: int = 0, b: int = 0, c: int = 0) -> int:
    return int(_L().syn_key(seed, a, b, c))


def normal_bf16(shape, k: int, sigma: float, first: int = 0, out: np.ndarray | None = None) -> np.ndarray:
    """bf16 bit patterns (uint16) of stream ``k`` elements [first, first+size)."""
    n = int(np.prod(shape))
    if out is None:
        out = np.empty(shape, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == n
    _L().syn_normal_bf16(out.ctypes.data, n, k, sigma, first)
    return out


def normal_bf16_mean(shape, k: int, mean: float, sigma: float) -> np.ndarray:
    """bf16 bit patterns of ``mean`` + stream ``k`` (the same normal values as
    ``normal_bf16``, offset before the rounding)."""
    out = np.empty(shape, dtype=np.uint16)
    _L().syn_normal_bf16_mean(out.ctypes.data, out.size, k, mean, sigma, 0)
    return out


def normal_f32(n: int, k: int, sigma: float) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _L().syn_normal_f32(out.ctypes.data, n, k, sigma)
    return out


def uniform_i32(n: int, k: int, lo: int, hi: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _L().syn_uniform_i32(out.ctypes.data, n, k, lo, hi)
    return out


def fill_bf16(shape, value: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    _L().syn_fill_bf16(out.ctypes.data, out.size, value)
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a bit shift)."""
    return (a.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class ModelShape:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float
    rope_theta: float
    tied: bool

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def n_params(self) -> int:
        H, F = self.hidden, self.ffn
        per_layer = 2 * H + H * (self.q_dim + 2 * self.kv_dim) + self.q_dim * H + 3 * H * F
        return self.vocab * H * (1 if self.tied else 2) + H + self.n_layers * per_layer


@dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    batch: int
    context: int            # KV positions already filled before the first decode step (per sequence, unless ragged)
    steps: int              # greedy decode steps
    ragged: tuple | None = None   # (lo, hi) inclusive: per-sequence context ~U[lo, hi]
    prompt: bool = False    # the context is a prompt the oracle prefills (tiny)

    def lengths(self) -> np.ndarray:
        """Per-sequence context length (= position of the first decode token)."""
        if self.ragged is None:
            return np.full(self.batch, self.context, dtype=np.int32)
        lo, hi = self.ragged
        return uniform_i32(self.batch, key(SEED_LENGTHS), lo, hi + 1)

    def max_seq(self) -> int:
        return int(self.lengths().max()) + self.steps


TINY = ModelShape(2, 256, 4, 2, 64, 1024, 4096, 1e-5, 1e4, True)
LLAMA_1B = ModelShape(16, 2048, 32, 8, 64, 8192, 128256, 1e-5, 5e5, True)
LLAMA_8B = ModelShape(32, 4096, 32, 8, 128, 14336, 128256, 1e-5, 5e5, False)

WORKLOADS = {
    "tiny": Workload("tiny", TINY, 1, 64, 16, prompt=True),
    "llama1b": Workload("llama1b", LLAMA_1B, 1, 1024, 128),
    "llama1b_8k": Workload("llama1b_8k", LLAMA_1B, 1, 8192, 64),
    "llama1b_b16": Workload("llama1b_b16", LLAMA_1B, 16, 0, 64, ragged=(512, 4096)),
    "llama8b": Workload("llama8b", LLAMA_8B, 1, 2048, 32),
}


def shape_dict(s: ModelShape) -> dict:
    return asdict(s)


# --------------------------------------------------------------------------
# Model weights: bf16 bit patterns in the plain [out][in] row-major layout.
# --------------------------------------------------------------------------

LAYER_TENSORS = ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")


def layer_tensor_shape(s: ModelShape, name: str):
    H, F = s.hidden, s.ffn
    return {
        "attn_norm": (H,), "ffn_norm": (H,),
        "wq": (s.q_dim, H), "wk": (s.kv_dim, H), "wv": (s.kv_dim, H),
        "wo": (H, s.q_dim),
        "w_gate": (F, H), "w_up": (F, H), "w_down": (H, F),
    }[name]


_KIND = {"wq": K_WQ, "wk": K_WK, "wv": K_WV, "wo": K_WO, "w_gate": K_WGATE, "w_up": K_WUP, "w_down": K_WDOWN}


def make_norm(s: ModelShape, kind: int, layer: int, norm_sigma: float = 0.0, seed: int = SEED_WEIGHTS) -> np.ndarray:
    """An RMSNorm weight vector: 1.0 everywhere (the workloads), or with
    ``norm_sigma`` > 0 seeded values ~N(1, norm_sigma) from stream
    key(seed, kind, layer)."""
    if norm_sigma <= 0:
        return fill_bf16((s.hidden,), 1.0)
    return normal_bf16_mean((s.hidden,), key(seed, kind, layer), 1.0, norm_sigma)


def make_layer_tensor(s: ModelShape, layer: int, name: str, seed: int = SEED_WEIGHTS, out=None,
                      norm_sigma: float = 0.0) -> np.ndarray:
    if name.endswith("norm"):
        return make_norm(s, K_ATTN_NORM if name == "attn_norm" else K_FFN_NORM, layer, norm_sigma, seed)
    shp = layer_tensor_shape(s, name)
    return normal_bf16(shp, key(seed, _KIND[name], layer), WEIGHT_SIGMA, out=out)


def make_embed(s: ModelShape, seed: int = SEED_WEIGHTS, out=None) -> np.ndarray:
    return normal_bf16((s.vocab, s.hidden), key(seed, K_EMBED, 0), WEIGHT_SIGMA, out=out)


def make_lm_head(s: ModelShape, seed: int = SEED_WEIGHTS, out=None) -> np.ndarray:
    """Untied LM head; for a tied model the head *is* the embedding."""
    return normal_bf16((s.vocab, s.hidden), key(seed, K_LM_HEAD, 0), WEIGHT_SIGMA, out=out)


def make_model(s: ModelShape, seed: int = SEED_WEIGHTS, norm_sigma: float = 0.0) -> dict:
    """All weights on the host: {'embed', 'lm_head', 'final_norm', 'layers': [dict]}.
    Norm weights are 1.0 unless ``norm_sigma`` > 0 (then ~N(1, norm_sigma),
    a distinct seeded vector per norm and layer)."""
    embed = make_embed(s, seed)
    m = {
        "embed": embed,
        "lm_head": embed if s.tied else make_lm_head(s, seed),
        "final_norm": make_norm(s, K_FINAL_NORM, 0, norm_sigma, seed),
        "layers": [{n: make_layer_tensor(s, l, n, seed, norm_sigma=norm_sigma) for n in LAYER_TENSORS}
                   for l in range(s.n_layers)],
    }
    return m


def with_norms(model: dict, s: ModelShape, norm_sigma: float, seed: int = SEED_WEIGHTS) -> dict:
    """A shallow copy of ``model`` whose norm weights are replaced by the
    ~N(1, norm_sigma) vectors ``make_model(..., norm_sigma)`` would make (the
    large matrices are shared, not copied)."""
    layers = []
    for l, L in enumerate(model["layers"]):
        d = dict(L)
        d["attn_norm"] = make_norm(s, K_ATTN_NORM, l, norm_sigma, seed)
        d["ffn_norm"] = make_norm(s, K_FFN_NORM, l, norm_sigma, seed)
        layers.append(d)
    out = dict(model)
    out["layers"] = layers
    out["final_norm"] = make_norm(s, K_FINAL_NORM, 0, norm_sigma, seed)
    return out


# --------------------------------------------------------------------------
# KV cache prefix, layout [layer][batch][kv_head][max_seq][head_dim] (bf16)
# --------------------------------------------------------------------------

def kv_key(seed: int, which: int, layer: int, b: int, g: int) -> int:
    return key(seed, which * 65536 + layer, b, g)


def fill_kv_prefix(s: ModelShape, kcache: np.ndarray, vcache: np.ndarray, lengths, seed: int = SEED_KV):
    """Fill positions [0, lengths[b]) of every (layer, b, kv head) with N(0,1) bf16.

    The values stand for post-RoPE keys and for values of earlier tokens."""
    L, B, G, S, d = kcache.shape
    for l in range(L):
        for b in range(B):
            n = int(lengths[b])
            for g in range(G):
                for which, cache in ((0, kcache), (1, vcache)):
                    blk = np.empty((n, d), dtype=np.uint16)
                    normal_bf16((n, d), kv_key(seed, which, l, b, g), KV_SIGMA, out=blk)
                    cache[l, b, g, :n, :] = blk


def alloc_kv(s: ModelShape, batch: int, max_seq: int):
    shp = (s.n_layers, batch, s.n_kv_heads, max_seq, s.head_dim)
    return np.zeros(shp, dtype=np.uint16), np.zeros(shp, dtype=np.uint16)


def first_tokens(w: Workload) -> np.ndarray:
    """Token id fed to the first decode step of each sequence."""
    return uniform_i32(w.batch, key(SEED_TOKENS, 0), 0, w.shape.vocab)


def prompt_tokens(w: Workload, b: int = 0) -> np.ndarray:
    """Random prompt (tiny workload): ``context`` ids uniform over the vocabulary."""
    return uniform_i32(w.context, key(SEED_TOKENS, 1, b), 0, w.shape.vocab)
