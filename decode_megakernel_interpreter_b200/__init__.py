"""Python binding of libmk.so, the decode megakernel engine (C ABI in
include/mk.h and include/mk_host.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libmk.so.  PyTorch supplies device memory and streams.  The
functions keep the C names (``mk_create``, ``mk_plan``, ``mk_decode_step``,
``mk_get_status``, ``mk_status_string``, ``mk_destroy``, ...); ``Engine`` wraps
them for torch tensors.  If libmk.so is missing, loading raises: there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmk.so")

MK_OK = 0
MK_ERR_INVALID_ARG = -1
MK_ERR_UNSUPPORTED_SHAPE = -2
MK_ERR_NOT_PLANNED = -3
MK_ERR_CUDA = -4
MK_ERR_LAUNCH = -5
MK_ERR_TIMEOUT = -6
MK_ERR_DEVICE_INPUT = -7
MK_ERR_OUT_OF_MEMORY = -8

MK_SCHED_STATIC, MK_SCHED_DYNAMIC, MK_SCHED_EVENT = 0, 1, 2
MK_EXEC_MEGAKERNEL, MK_EXEC_PER_OP, MK_EXEC_PER_OP_GRAPH, MK_EXEC_MEGAKERNEL_GENERIC = 0, 1, 2, 3
MK_TRACE_WORDS = 12

OP_NAMES = {0: "nop", 1: "qkv", 2: "attn", 3: "oproj", 4: "gateup", 5: "down", 6: "lmhead"}


class MkError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {mk_status_string(code)} ({code})")


class mk_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_double),
                ("tied_lm_head", ctypes.c_int32), ("max_batch", ctypes.c_int32), ("max_seq", ctypes.c_int32)]


class mk_layer_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")]


class mk_weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("layers", ctypes.POINTER(mk_layer_weights))]


class mk_kv_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p)]


class mk_plan_opts(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("kv_splits", ctypes.c_int32), ("sched_mode", ctypes.c_int32),
                ("exec_mode", ctypes.c_int32), ("num_sms", ctypes.c_int32), ("trace", ctypes.c_int32),
                ("wait_timeout_ns", ctypes.c_int64), ("l2_prefetch_kb", ctypes.c_int32),
                ("debug_drop_producer", ctypes.c_int32), ("max_inflight_pages", ctypes.c_int32),
                ("tensor_qkv_o", ctypes.c_int32), ("use_tcgen05", ctypes.c_int32)]


class mk_plan_info(ctypes.Structure):
    _fields_ = [("num_ctas", ctypes.c_int32), ("threads_per_cta", ctypes.c_int32), ("smem_bytes", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("num_instructions", ctypes.c_int32),
                ("num_counters", ctypes.c_int32), ("kv_splits", ctypes.c_int32), ("max_queue_len", ctypes.c_int32),
                ("weight_bytes_per_step", ctypes.c_int64), ("kernel_variant", ctypes.c_int32),
                ("estimated_step_us", ctypes.c_int32)]


class mk_instr_desc(ctypes.Structure):
    _fields_ = [("op", ctypes.c_uint8), ("pad", ctypes.c_uint8), ("layer", ctypes.c_uint16),
                ("a", ctypes.c_uint32), ("b", ctypes.c_uint32), ("c", ctypes.c_uint32),
                ("wait_ctr", ctypes.c_uint32), ("wait_cnt", ctypes.c_uint32), ("sig_ctr", ctypes.c_uint32),
                ("sig_n", ctypes.c_uint16), ("seq", ctypes.c_uint16)]


class mk_cost_params(ctypes.Structure):
    _fields_ = [("sm_gbs", ctypes.c_double), ("ring_pages", ctypes.c_int32), ("exchange_us", ctypes.c_double),
                ("page_us", ctypes.c_double), ("attn_page_us", ctypes.c_double), ("attn_fixed_us", ctypes.c_double),
                ("merge_us", ctypes.c_double), ("instr_us", ctypes.c_double), ("launch_us", ctypes.c_double),
                ("tc_page_us", ctypes.c_double), ("cc_page_us_seq", ctypes.c_double), ("conv_ctas", ctypes.c_int32),
                ("merge_split_us", ctypes.c_double)]


class mk_cost_estimate(ctypes.Structure):
    _fields_ = [("step_us", ctypes.c_double), ("per_op_us", ctypes.c_double), ("hbm_floor_us", ctypes.c_double),
                ("savings_us", ctypes.c_double), ("stage_us", ctypes.c_double * 7)]


_lib = None


def load(path: str = LIB_PATH):
    """Load libmk.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m decode_megakernel_interpreter_b200.build`")
    L = ctypes.CDLL(path)
    vp, i32, i64, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    P = ctypes.POINTER
    L.mk_create.restype = i32
    L.mk_create.argtypes = [P(mk_config), P(mk_weights), P(mk_kv_cache), P(vp)]
    L.mk_plan.restype = i32
    L.mk_plan.argtypes = [vp, P(mk_plan_opts)]
    L.mk_decode_step.restype = i32
    L.mk_decode_step.argtypes = [vp, vp, vp, vp, vp, vp]
    L.mk_prefill.restype = i32
    L.mk_prefill.argtypes = [vp, i32, vp, i32, i32, vp, vp, vp]
    L.mk_tp_create.restype = i32
    L.mk_tp_create.argtypes = [P(mk_config), P(mk_weights), P(mk_kv_cache), i32, P(vp)]
    L.mk_tp_plan.restype = i32
    L.mk_tp_plan.argtypes = [vp, P(mk_plan_opts)]
    L.mk_tp_decode_step.restype = i32
    L.mk_tp_decode_step.argtypes = [vp, vp, vp, vp, vp, vp]
    L.mk_tp_get_status.restype = i32
    L.mk_tp_get_status.argtypes = [vp, vp]
    L.mk_tp_destroy.restype = None
    L.mk_tp_destroy.argtypes = [vp]
    L.mk_get_status.restype = i32
    L.mk_get_status.argtypes = [vp, vp]
    L.mk_status_string.restype = ctypes.c_char_p
    L.mk_status_string.argtypes = [i32]
    L.mk_destroy.restype = None
    L.mk_destroy.argtypes = [vp]
    L.mk_get_error_detail.restype = i32
    L.mk_get_error_detail.argtypes = [vp, P(i32)]
    L.mk_get_plan_info.restype = i32
    L.mk_get_plan_info.argtypes = [vp, P(mk_plan_info)]
    L.mk_trace_read.restype = i32
    L.mk_trace_read.argtypes = [vp, P(ctypes.c_uint64), sz]
    L.mk_host_plan.restype = i32
    L.mk_host_plan.argtypes = [P(mk_config), P(mk_plan_opts), i32, P(mk_instr_desc), i32, P(i32), P(i32), P(i32),
                               P(mk_plan_info), ctypes.c_char_p, sz]
    L.mk_noalloc_get_status.restype = i32
    L.mk_noalloc_get_status.argtypes = [vp, vp]
    L.mk_decode_step_noalloc.restype = i32
    L.mk_decode_step_noalloc.argtypes = [P(mk_config), P(mk_weights), P(mk_kv_cache), vp, vp, vp, vp, vp]
    L.mk_cost_params_default.restype = None
    L.mk_cost_params_default.argtypes = [P(mk_cost_params)]
    L.mk_host_plan_estimate.restype = i32
    L.mk_host_plan_estimate.argtypes = [P(mk_config), P(mk_plan_opts), i32, i32, P(mk_cost_params),
                                        P(mk_cost_estimate), ctypes.c_char_p, sz]
    L.mk_host_plan_simulate.restype = i32
    L.mk_host_plan_simulate.argtypes = [P(mk_config), P(mk_plan_opts), i32, i32, u64, i32, ctypes.c_char_p, sz]
    _lib = L
    return L


# ---------------------------------------------------------------- C names

def mk_status_string(code: int) -> str:
    return load().mk_status_string(int(code)).decode()


def mk_create(cfg: mk_config, weights: mk_weights, kv: mk_kv_cache) -> int:
    h = ctypes.c_void_p()
    rc = load().mk_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(kv), ctypes.byref(h))
    if rc != MK_OK:
        raise MkError(rc, "mk_create")
    return h.value


def mk_plan(h: int, opts: mk_plan_opts | None) -> None:
    rc = load().mk_plan(h, ctypes.byref(opts) if opts is not None else None)
    if rc != MK_OK:
        raise MkError(rc, "mk_plan")


def mk_decode_step(h: int, tokens: int, positions: int, logits_out: int | None, next_tokens_out: int,
                   stream: int | None) -> int:
    """Raw pointers (ints).  Returns the status code (no exception: the step is async)."""
    return load().mk_decode_step(h, tokens, positions, logits_out, next_tokens_out, stream)


def mk_prefill(h: int, seq: int, tokens: int, n_tokens: int, pos0: int, logits_out: int | None,
               next_token_out: int, stream: int | None) -> int:
    """Raw pointers (ints).  Returns the status code (asynchronous)."""
    return load().mk_prefill(h, seq, tokens, n_tokens, pos0, logits_out, next_token_out, stream)


def mk_decode_step_noalloc(cfg: mk_config, weights: mk_weights, kv: mk_kv_cache, tokens: int, positions: int,
                           logits_out: int | None, next_tokens_out: int, stream: int | None) -> int:
    """The allocation-free step (scratch in a fixed device array; see mk.h).
    Raw pointers (ints); returns the status code."""
    return load().mk_decode_step_noalloc(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(kv), tokens,
                                         positions, logits_out, next_tokens_out, stream)


def mk_noalloc_get_status(stream: int | None) -> tuple:
    """(status code, detail words) of the last allocation-free call on the current device."""
    d = (ctypes.c_int32 * 6)()
    rc = load().mk_noalloc_get_status(stream, d)
    return rc, list(d)


def mk_get_status(h: int, stream: int | None) -> int:
    return load().mk_get_status(h, stream)


def mk_destroy(h: int) -> None:
    load().mk_destroy(h)


def mk_get_error_detail(h: int) -> list:
    d = (ctypes.c_int32 * 6)()
    rc = load().mk_get_error_detail(h, d)
    if rc != MK_OK:
        raise MkError(rc, "mk_get_error_detail")
    return list(d)


def mk_get_plan_info(h: int) -> mk_plan_info:
    info = mk_plan_info()
    rc = load().mk_get_plan_info(h, ctypes.byref(info))
    if rc != MK_OK:
        raise MkError(rc, "mk_get_plan_info")
    return info


def mk_trace_read(h: int, n_instr: int):
    import numpy as np
    out = np.zeros((n_instr, MK_TRACE_WORDS), dtype=np.uint64)
    rc = load().mk_trace_read(h, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64)), out.size)
    if rc != MK_OK:
        raise MkError(rc, "mk_trace_read")
    return out


def mk_host_plan(cfg: mk_config, opts: mk_plan_opts | None, num_ctas: int):
    """Host-only plan: (instructions as a structured list, queue_off, queue_len, info)."""
    L = load()
    n = ctypes.c_int32()
    err = ctypes.create_string_buffer(512)
    info = mk_plan_info()
    o = ctypes.byref(opts) if opts is not None else None
    rc = L.mk_host_plan(ctypes.byref(cfg), o, num_ctas, None, 0, ctypes.byref(n), None, None, ctypes.byref(info), err, 512)
    if rc != MK_OK:
        raise MkError(rc, "mk_host_plan: " + err.value.decode())
    arr = (mk_instr_desc * n.value)()
    off = (ctypes.c_int32 * num_ctas)()
    ln = (ctypes.c_int32 * num_ctas)()
    rc = L.mk_host_plan(ctypes.byref(cfg), o, num_ctas, arr, n.value, ctypes.byref(n), off, ln, ctypes.byref(info),
                        err, 512)
    if rc != MK_OK:
        raise MkError(rc, "mk_host_plan: " + err.value.decode())
    return list(arr), list(off), list(ln), info


def mk_host_plan_simulate(cfg: mk_config, opts: mk_plan_opts | None, num_ctas: int, steps: int, seed: int,
                          timeout_ms: int = 5000) -> str:
    """'' if the simulated plan is race- and deadlock-free, else the failure."""
    err = ctypes.create_string_buffer(1024)
    rc = load().mk_host_plan_simulate(ctypes.byref(cfg), ctypes.byref(opts) if opts is not None else None, num_ctas,
                                      steps, seed, timeout_ms, err, 1024)
    return "" if rc == MK_OK else (err.value.decode() or mk_status_string(rc))


def mk_cost_params_default() -> mk_cost_params:
    q = mk_cost_params()
    load().mk_cost_params_default(ctypes.byref(q))
    return q


def mk_host_plan_estimate(cfg: mk_config, opts: mk_plan_opts | None, num_ctas: int, context: int,
                          params: mk_cost_params | None = None) -> mk_cost_estimate:
    """The cost model's estimate of a plan (see mk_host.h)."""
    out = mk_cost_estimate()
    err = ctypes.create_string_buffer(512)
    rc = load().mk_host_plan_estimate(ctypes.byref(cfg), ctypes.byref(opts) if opts is not None else None, num_ctas,
                                      context, ctypes.byref(params) if params is not None else None,
                                      ctypes.byref(out), err, 512)
    if rc != MK_OK:
        raise MkError(rc, "mk_host_plan_estimate: " + err.value.decode())
    return out


# ---------------------------------------------------------------- torch wrapper

def make_config(shape, max_batch: int, max_seq: int) -> mk_config:
    """mk_config from a shape object/dict (n_layers, hidden, n_q_heads,
    n_kv_heads, head_dim, ffn, vocab, rms_eps, rope_theta, tied)."""
    g = (lambda k: shape[k]) if isinstance(shape, dict) else (lambda k: getattr(shape, k))
    return mk_config(g("n_layers"), g("hidden"), g("n_q_heads"), g("n_kv_heads"), g("head_dim"), g("ffn"),
                     g("vocab"), float(g("rms_eps")), float(g("rope_theta")), int(bool(g("tied"))), max_batch,
                     max_seq)


def plan_opts(batch: int = 1, kv_splits: int = 0, sched: str = "static", exec_mode: str = "megakernel",
              num_sms: int = 0, trace: bool = False, wait_timeout_ns: int = 0, l2_prefetch_kb: int = 0,
              debug_drop_producer: bool = False, max_inflight_pages: int = 0,
              tensor_qkv_o: bool = False, use_tcgen05: int = 0) -> mk_plan_opts:
    return mk_plan_opts(batch, kv_splits, {"static": 0, "dynamic": 1, "event": 2}[sched],
                        {"megakernel": 0, "per_op": 1, "per_op_graph": 2, "megakernel_generic": 3}[exec_mode], num_sms, int(trace),
                        wait_timeout_ns, l2_prefetch_kb, int(debug_drop_producer), max_inflight_pages,
                        int(tensor_qkv_o), int(use_tcgen05))


def _abi_model(weights: dict, kcache, vcache):
    """The C structs (layer array, mk_weights, mk_kv_cache) over torch tensors;
    the layer array must stay referenced while the structs are used."""
    layers = weights["layers"]
    lw = (mk_layer_weights * len(layers))()
    for i, L in enumerate(layers):
        for n, _ in mk_layer_weights._fields_:
            setattr(lw[i], n, _ptr(L[n]))
    lm = weights.get("lm_head")
    w = mk_weights(_ptr(weights["embed"]), _ptr(lm) if lm is not None else None, _ptr(weights["final_norm"]), lw)
    return lw, w, mk_kv_cache(_ptr(kcache), _ptr(vcache))


class Engine:
    """Owns an mk handle over torch CUDA tensors.

    weights: dict with 'embed', 'lm_head' (or None when tied), 'final_norm'
    and 'layers' (list of dicts: attn_norm, wq, wk, wv, wo, ffn_norm, w_gate,
    w_up, w_down), all contiguous torch.bfloat16 (or int16/uint16 bit
    pattern) CUDA tensors in [out][in] layout.  kcache / vcache:
    [n_layers][max_batch][n_kv_heads][max_seq][head_dim] bf16 CUDA tensors.
    The tensors are borrowed and must outlive the engine."""

    def __init__(self, shape, weights: dict, kcache, vcache, max_batch: int, max_seq: int):
        self.cfg = make_config(shape, max_batch, max_seq)
        self._keep = (weights, kcache, vcache)
        self._lw, self._w, self._kv = _abi_model(weights, kcache, vcache)
        self.h = mk_create(self.cfg, self._w, self._kv)
        self.info = None

    def plan(self, **kw) -> mk_plan_info:
        self.opts = plan_opts(**kw)
        mk_plan(self.h, self.opts)
        self.info = mk_get_plan_info(self.h)
        return self.info

    def decode_step(self, tokens, positions, logits_out, next_tokens_out, stream=None) -> None:
        import torch
        s = stream if stream is not None else torch.cuda.current_stream()
        rc = mk_decode_step(self.h, _ptr(tokens), _ptr(positions), _ptr(logits_out) if logits_out is not None else None,
                            _ptr(next_tokens_out), s.cuda_stream)
        if rc != MK_OK:
            raise MkError(rc, "mk_decode_step")

    def prefill(self, seq, tokens, pos0, logits_out, next_token_out, stream=None) -> None:
        """Prompt tokens (device int32 tensor) of sequence `seq` from position
        pos0: their K/V rows, and the last token's logits / greedy next token."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream()
        rc = mk_prefill(self.h, seq, _ptr(tokens), int(tokens.numel()), pos0,
                        _ptr(logits_out) if logits_out is not None else None, _ptr(next_token_out), s.cuda_stream)
        if rc != MK_OK:
            raise MkError(rc, "mk_prefill")

    def status(self, stream=None) -> int:
        import torch
        s = stream if stream is not None else torch.cuda.current_stream()
        return mk_get_status(self.h, s.cuda_stream)

    def trace(self):
        return mk_trace_read(self.h, self.info.num_instructions)

    def close(self) -> None:
        if getattr(self, "h", None):
            mk_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    assert t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors"
    return t.data_ptr()


class TpEngine:
    """A tensor-parallel group of n ranks emulated on this GPU (mk_tp_*): the
    same weights / cache arguments as Engine (batch 1 plans)."""

    def __init__(self, shape, weights: dict, kcache, vcache, max_batch: int, max_seq: int, n_ranks: int):
        self.cfg = make_config(shape, max_batch, max_seq)
        self._keep = (weights, kcache, vcache)
        self._lw, self._w, self._kv = _abi_model(weights, kcache, vcache)
        g = ctypes.c_void_p()
        rc = load().mk_tp_create(ctypes.byref(self.cfg), ctypes.byref(self._w), ctypes.byref(self._kv), n_ranks,
                                 ctypes.byref(g))
        if rc != MK_OK:
            raise MkError(rc, "mk_tp_create")
        self.g = g.value
        self.n_ranks = n_ranks

    def plan(self, **kw) -> None:
        self.opts = plan_opts(**kw)
        rc = load().mk_tp_plan(self.g, ctypes.byref(self.opts))
        if rc != MK_OK:
            raise MkError(rc, "mk_tp_plan")

    def decode_step(self, tokens, positions, logits_out, next_tokens_out, stream=None) -> None:
        import torch
        s = stream if stream is not None else torch.cuda.current_stream()
        rc = load().mk_tp_decode_step(self.g, _ptr(tokens), _ptr(positions),
                                      _ptr(logits_out) if logits_out is not None else None, _ptr(next_tokens_out),
                                      s.cuda_stream)
        if rc != MK_OK:
            raise MkError(rc, "mk_tp_decode_step")

    def status(self, stream=None) -> int:
        import torch
        s = stream if stream is not None else torch.cuda.current_stream()
        return load().mk_tp_get_status(self.g, s.cuda_stream)

    def close(self) -> None:
        if getattr(self, "g", None):
            load().mk_tp_destroy(self.g)
            self.g = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
