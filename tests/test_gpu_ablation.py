"""The ablation measurement tool runs end to end and its numbers are consistent.

Tiny workload (all query blocks): every variant's output is finite; no top-s choice
keeps more dense attention mass than the oracle top-k by mass; with s = nK every
variant keeps all the mass.
"""

import math

import pytest

from ablation_report import VARIANTS, markdown, run_ablation

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("workload", ["tiny", "tiny_dense"])
def test_ablation_tiny(workload):
    rep = run_ablation(workload, blocks=64, head=0)
    v = rep["variants"]
    assert set(v) == {n for n, _, _ in VARIANTS} | {"topk_oracle_mass"}
    best = v["topk_oracle_mass"]["mass_captured"]
    for name, m in v.items():
        assert math.isfinite(m["rel_l2_err"]) and 0.0 <= m["mass_captured"] <= 1.0 + 1e-9
        assert m["mass_captured"] <= best + 1e-9, name
    if rep["s"] == rep["nK"]:
        for m in v.values():
            assert abs(m["mass_captured"] - 1.0) < 1e-9
            assert m["rel_l2_err"] < 1e-2  # bf16 inputs/outputs against fp64
    assert "variant" in markdown(rep)
