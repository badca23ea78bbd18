"""Plumbing between host-side bf16 bit-pattern arrays (numpy uint16) and the
engine's torch CUDA tensors: uploading a model and a KV cache, and building an
Engine for a named workload.  No arithmetic of the decode step lives here."""
from __future__ import annotations

import numpy as np
import torch

from . import Engine

LAYER_TENSORS = ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")


def to_device_bf16(a: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 CUDA tensor (same bytes)."""
    assert a.dtype == np.uint16
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.to(device, non_blocking=False).view(torch.bfloat16)


def upload_model(host: dict, tied: bool, device="cuda") -> dict:
    dev = {
        "embed": to_device_bf16(host["embed"], device),
        "final_norm": to_device_bf16(host["final_norm"], device),
        "layers": [{n: to_device_bf16(L[n], device) for n in LAYER_TENSORS} for L in host["layers"]],
    }
    dev["lm_head"] = None if tied else to_device_bf16(host["lm_head"], device)
    return dev


def upload_kv(k: np.ndarray, v: np.ndarray, device="cuda"):
    return to_device_bf16(k, device), to_device_bf16(v, device)


def kv_to_host(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def make_engine(shape, dev_model: dict, kc: torch.Tensor, vc: torch.Tensor, max_batch: int, max_seq: int) -> Engine:
    return Engine(shape, dev_model, kc, vc, max_batch, max_seq)


def kv_row_to_host(t: torch.Tensor, b: int, p: int) -> np.ndarray:
    """Row p of sequence b of a [L][B][n_kv][max_seq][d] cache: [L][n_kv][d]."""
    return t[:, b, :, p].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def replace_norms(dev: dict, host: dict, device="cuda") -> dict:
    """A device model sharing every matrix of `dev`, with the norm vectors
    uploaded from `host`."""
    out = dict(dev)
    out["final_norm"] = to_device_bf16(host["final_norm"], device)
    out["layers"] = []
    for Ld, Lh in zip(dev["layers"], host["layers"]):
        d = dict(Ld)
        d["attn_norm"] = to_device_bf16(Lh["attn_norm"], device)
        d["ffn_norm"] = to_device_bf16(Lh["ffn_norm"], device)
        out["layers"].append(d)
    return out
