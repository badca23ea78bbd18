"""The oracle against its stored regression record (tests/golden): the
greedy tokens exactly, the logits to fp64 rounding."""
import importlib.util
import json
import os

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


def _maker():
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(GOLDEN, "make_golden.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_tiny_greedy_record_unchanged():
    with open(os.path.join(GOLDEN, "tiny_greedy_f64.json")) as f:
        want = json.load(f)
    got = _maker().tiny_greedy_record()
    assert [i for i, _ in got["prompt_top5"]] == [i for i, _ in want["prompt_top5"]]
    for (_, a), (_, b) in zip(got["prompt_top5"], want["prompt_top5"]):
        assert a == pytest.approx(b, rel=1e-12, abs=1e-12)
    assert len(got["steps"]) == len(want["steps"]) == 16
    for g, w in zip(got["steps"], want["steps"]):
        assert (g["token_in"], g["pos"], g["next"]) == (w["token_in"], w["pos"], w["next"])
        for key in ("max", "margin", "sum"):
            assert g[key] == pytest.approx(w[key], rel=1e-12, abs=1e-11), key
