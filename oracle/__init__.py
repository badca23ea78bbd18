"""CPU oracle of one Llama-style decode step (ctypes wrapper over liboracle.so).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  It shares no
code with the GPU engine and never calls it.

Two precisions are built from one C body: ``"f64"`` (double arithmetic, the
definition the GPU is compared against) and ``"f32"`` (float arithmetic with
sequential accumulation, used to bound fp32 rounding).  Weights and the KV
cache are numpy ``uint16`` arrays of bf16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, f) for f in ("llama_oracle.c", "llama_oracle_body.h", "llama_oracle.h")]
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to this file (gcc, OpenMP over output rows)."""
    newest = max(os.path.getmtime(s) for s in _SRCS)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + ".tmp"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRCS[0], "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab")] + \
               [("rms_eps", ctypes.c_double), ("rope_theta", ctypes.c_double)]


class _Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")]


class _Model(ctypes.Structure):
    _fields_ = [("shape", _Shape), ("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("final_norm", ctypes.c_void_p), ("layers", ctypes.POINTER(_Layer))]


class _KV(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("layer_stride", ctypes.c_int64), ("head_stride", ctypes.c_int64)]


class _Dump(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q", "k", "v", "attn", "x_attn", "act", "x_out", "final_a")]


_lib = None


def lib():
    """The oracle library: liboracle.so (built on first use), or the library
    named by MK_ORACLE_LIB (the planted-mistake test loads mutated builds of
    the same source that way)."""
    global _lib
    if _lib is None:
        L = ctypes.CDLL(os.environ.get("MK_ORACLE_LIB") or build())
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        for sfx, real in (("_f64", ctypes.c_double), ("_f32", ctypes.c_float)):
            getattr(L, "orc_bf16_to_real" + sfx).restype = real
            getattr(L, "orc_bf16_to_real" + sfx).argtypes = [ctypes.c_uint16]
            getattr(L, "orc_real_to_bf16" + sfx).restype = ctypes.c_uint16
            getattr(L, "orc_real_to_bf16" + sfx).argtypes = [real]
            getattr(L, "orc_matvec" + sfx).argtypes = [vp, vp, i32, i32, vp]
            getattr(L, "orc_rmsnorm" + sfx).argtypes = [vp, vp, i32, dbl, vp]
            getattr(L, "orc_rope" + sfx).argtypes = [vp, i32, i32, dbl]
            getattr(L, "orc_attention_head" + sfx).argtypes = [vp, vp, vp, i32, i32, vp]
            getattr(L, "orc_silu" + sfx).restype = real
            getattr(L, "orc_silu" + sfx).argtypes = [real]
            getattr(L, "orc_decode_step" + sfx).argtypes = [ctypes.POINTER(_Model), ctypes.POINTER(_KV), i32, i32, vp,
                                                          ctypes.POINTER(_Dump)]
            getattr(L, "orc_prefill" + sfx).argtypes = [ctypes.POINTER(_Model), ctypes.POINTER(_KV), vp, i32, vp, vp]
        L.orc_argmax.restype = i32
        L.orc_argmax.argtypes = [vp, i32]
        _lib = L
    return _lib


def _dt(precision):
    return {"f64": np.float64, "f32": np.float32}[precision]


def _ptr(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data


# ---------------------------------------------------------------- primitives

def bf16_to_real(b: int, precision="f64") -> float:
    return getattr(lib(), "orc_bf16_to_real_" + precision)(b)


def real_to_bf16(x: float, precision="f64") -> int:
    return int(getattr(lib(), "orc_real_to_bf16_" + precision)(x))


def matvec(W: np.ndarray, x: np.ndarray, precision="f64") -> np.ndarray:
    W = np.ascontiguousarray(W, dtype=np.uint16)
    x = np.ascontiguousarray(x, dtype=_dt(precision))
    y = np.empty(W.shape[0], dtype=_dt(precision))
    getattr(lib(), "orc_matvec_" + precision)(_ptr(W), _ptr(x), W.shape[0], W.shape[1], _ptr(y))
    return y


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float, precision="f64") -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=_dt(precision))
    gamma = np.ascontiguousarray(gamma, dtype=np.uint16)
    y = np.empty_like(x)
    getattr(lib(), "orc_rmsnorm_" + precision)(_ptr(x), _ptr(gamma), x.size, eps, _ptr(y))
    return y


def rope(v: np.ndarray, pos: int, theta: float, precision="f64") -> np.ndarray:
    v = np.array(v, dtype=_dt(precision), copy=True)
    getattr(lib(), "orc_rope_" + precision)(_ptr(v), v.size, pos, theta)
    return v


def attention_head(q: np.ndarray, K: np.ndarray, V: np.ndarray, precision="f64") -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=_dt(precision))
    K = np.ascontiguousarray(K, dtype=np.uint16)
    V = np.ascontiguousarray(V, dtype=np.uint16)
    o = np.empty(q.size, dtype=_dt(precision))
    getattr(lib(), "orc_attention_head_" + precision)(_ptr(q), _ptr(K), _ptr(V), K.shape[0], q.size, _ptr(o))
    return o


def silu(z: float, precision="f64") -> float:
    return getattr(lib(), "orc_silu_" + precision)(z)


def argmax(x: np.ndarray) -> int:
    x = np.ascontiguousarray(x, dtype=np.float64)
    return int(lib().orc_argmax(_ptr(x), x.size))


# ---------------------------------------------------------------- the model

class Oracle:
    """Decode steps of one model on the CPU.

    ``shape``: object or dict with n_layers, hidden, n_q_heads, n_kv_heads,
    head_dim, ffn, vocab, rms_eps, rope_theta.  ``model``: dict with 'embed',
    'lm_head', 'final_norm' and 'layers' (list of dicts of bf16 arrays in
    [out][in] layout).  The arrays are referenced, not copied.
    """

    def __init__(self, shape, model: dict, precision: str = "f64"):
        g = (lambda k: shape[k]) if isinstance(shape, dict) else (lambda k: getattr(shape, k))
        self.precision = precision
        self.vocab = int(g("vocab"))
        self.n_layers = int(g("n_layers"))
        self.hidden, self.ffn = int(g("hidden")), int(g("ffn"))
        self.q_dim = int(g("n_q_heads")) * int(g("head_dim"))
        self.kv_dim = int(g("n_kv_heads")) * int(g("head_dim"))
        self._keep = model
        self._layers = (_Layer * self.n_layers)()
        for i, L in enumerate(model["layers"]):
            for n, _ in _Layer._fields_:
                a = L[n]
                assert a.dtype == np.uint16 and a.flags.c_contiguous
                setattr(self._layers[i], n, a.ctypes.data)
        sh = _Shape(*[int(g(n)) for n in ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab")],
                    float(g("rms_eps")), float(g("rope_theta")))
        for n in ("embed", "lm_head", "final_norm"):
            assert model[n].dtype == np.uint16 and model[n].flags.c_contiguous
        self._model = _Model(sh, model["embed"].ctypes.data, model["lm_head"].ctypes.data,
                             model["final_norm"].ctypes.data, self._layers)

    @staticmethod
    def _kv(kcache: np.ndarray, vcache: np.ndarray, b: int) -> _KV:
        """kcache/vcache: [layer][batch][kv_head][max_seq][head_dim] uint16."""
        assert kcache.shape == vcache.shape and kcache.dtype == np.uint16 and kcache.flags.c_contiguous
        L, B, G, S, d = kcache.shape
        off = b * G * S * d * 2
        return _KV(kcache.ctypes.data + off, vcache.ctypes.data + off, B * G * S * d, S * d)

    def decode_step(self, kcache, vcache, b: int, token: int, pos: int, dump: bool = False):
        """Logits (float64 [vocab]) of sequence ``b``'s token at ``pos``; writes
        its K/V rows into the caches.  With ``dump`` also returns a dict of the
        per-stage values."""
        kv = self._kv(kcache, vcache, b)
        logits = np.empty(self.vocab, dtype=np.float64)
        d = None
        dp = None
        if dump:
            L, H, F, qd, kvd = self.n_layers, self.hidden, self.ffn, self.q_dim, self.kv_dim
            d = {"q": np.zeros((L, qd)), "k": np.zeros((L, kvd)), "v": np.zeros((L, kvd)),
                 "attn": np.zeros((L, qd)), "x_attn": np.zeros((L, H)), "act": np.zeros((L, F)),
                 "x_out": np.zeros((L, H)), "final_a": np.zeros(H)}
            dp = _Dump(*[d[n].ctypes.data for n, _ in _Dump._fields_])
        rc = getattr(lib(), "orc_decode_step_" + self.precision)(
            ctypes.byref(self._model), ctypes.byref(kv), int(token), int(pos), logits.ctypes.data,
            ctypes.byref(dp) if dp is not None else None)
        if rc != 0:
            raise ValueError("oracle decode_step: bad argument")
        return (logits, d) if dump else logits

    def prefill(self, kcache, vcache, b: int, tokens, all_logits: bool = False):
        """Full causal forward over ``tokens`` at positions 0..n-1 (fills the
        cache).  Returns the last position's logits, or all of them."""
        tokens = np.ascontiguousarray(tokens, dtype=np.int32)
        n = tokens.size
        kv = self._kv(kcache, vcache, b)
        last = np.empty(self.vocab, dtype=np.float64)
        allp = np.empty((n, self.vocab), dtype=np.float64) if all_logits else None
        rc = getattr(lib(), "orc_prefill_" + self.precision)(
            ctypes.byref(self._model), ctypes.byref(kv), tokens.ctypes.data, n,
            allp.ctypes.data if allp is not None else None, last.ctypes.data)
        if rc != 0:
            raise ValueError("oracle prefill: bad argument")
        return allp if all_logits else last
