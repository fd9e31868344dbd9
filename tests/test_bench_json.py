"""bench.py prints strict JSON: non-finite numbers (the stages a stage-only run does not
time) become null."""

import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _strict(text):
    def reject(name):
        raise ValueError(f"non-standard JSON constant {name}")
    return json.loads(text, parse_constant=reject)


def test_json_line_replaces_non_finite_numbers():
    out = {"ms_per_attn_call": float("nan"), "roofline": {"achieved": float("inf"), "peak": 1614.1},
           "cases": [float("-inf"), 2, "x"], "config": {"workload": "wan14b"}}
    d = _strict(_bench().json_line(out))
    assert d["ms_per_attn_call"] is None
    assert d["roofline"] == {"achieved": None, "peak": 1614.1}
    assert d["cases"] == [None, 2, "x"]
    assert d["config"] == {"workload": "wan14b"}
