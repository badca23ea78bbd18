"""Writes tests/golden/tiny_greedy_f64.json from the fp64 oracle alone.

The pages print no worked numeric example of the decode step, so the fixture
here is a regression record of the oracle itself on the tiny workload (2
layers, hidden 256, 4/2 heads of 64, ffn 1024, vocab 4096, theta 1e4, tied
head; 64-token seeded prompt, 16 greedy decode steps).  It calls only
``oracle`` and the seeded input generators in ``synth``; nothing in it comes
from the CUDA path.  Run from the repository root:

    python tests/golden/make_golden.py
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

OUT = os.path.join(HERE, "tiny_greedy_f64.json")


def tiny_greedy_record() -> dict:
    w = synth.WORKLOADS["tiny"]
    s = w.shape
    model = synth.make_model(s)
    k, v = synth.alloc_kv(s, 1, w.context + w.steps)
    orc = oracle.Oracle(s, model, "f64")
    prompt = synth.prompt_tokens(w)
    logits = np.asarray(orc.prefill(k, v, 0, prompt), dtype=np.float64)
    top = np.argsort(-logits, kind="stable")[:5]
    rec = {"prompt_top5": [[int(i), float(logits[i])] for i in top], "steps": []}
    tok, pos = oracle.argmax(logits), w.context
    for _ in range(w.steps):
        lg = np.asarray(orc.decode_step(k, v, 0, tok, pos), dtype=np.float64)
        nxt = oracle.argmax(lg)
        srt = np.sort(lg)
        rec["steps"].append({"token_in": int(tok), "pos": int(pos), "next": int(nxt), "max": float(srt[-1]),
                             "margin": float(srt[-1] - srt[-2]), "sum": float(lg.sum())})
        tok, pos = nxt, pos + 1
    return rec


def main() -> None:
    rec = tiny_greedy_record()
    rec = {"about": "fp64 oracle on the tiny workload: prompt logits top-5 and 16 greedy decode steps; "
                    "written by tests/golden/make_golden.py (oracle and synth only)", **rec}
    with open(OUT, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print("wrote", OUT)


if __name__ == "__main__":
    main()
