"""bench.py's reference arm (the CPU oracle) keeps the JSON contract, on the tiny workload."""

import argparse

import bench


def test_reference_arm_json_line():
    args = argparse.Namespace(workload="tiny", steps=2, warmup=1, ref_seconds=1.0)
    out = bench.run_reference(args, world=1, rank=0)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["impl"] == "reference" and out["value"] > 0 and out["unit"] == bench.UNIT
    assert out["metric"] == bench.METRIC and out["steps"] == 2 and out["warmup"] == 1
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == out["value"] and cb["sample"]
    import os

    assert cb["cores"] == min(64, len(os.sched_getaffinity(0)))  # one oracle process per core
    e2e = out["e2e"]
    assert e2e["value"] == out["value"] and e2e["unit"] == out["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert "workload" in out["config"]


def test_reference_arm_other_ranks_do_nothing():
    args = argparse.Namespace(workload="tiny", steps=1, warmup=1)
    assert bench.run_reference(args, world=2, rank=1) is None


def test_oracle_threads_positive():
    assert bench.oracle_threads() >= 1
