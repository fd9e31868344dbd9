"""Golden values printed on the AB-Attention page (onedev.kr/papers/1521).

The experiments paragraph prints the sparsity reached with KV block 4 and query
block 128 on 720p latents.  The planner budget s (whole 128-token tiles of kept
blocks) must reproduce those figures to every printed digit.
"""

import os

from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, budget_blocks

HERE = os.path.dirname(__file__)


def _rows():
    with open(os.path.join(HERE, "golden", "sparsity.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, fr, r, c, pct = line.split()
                yield name, int(fr), int(r), int(c), float(pct)


def test_budget_reproduces_printed_sparsity():
    for name, fr, r, c, pct in _rows():
        N = fr * r * c
        nK = N // 4
        # keep fraction = 1 - printed sparsity; s rounded down to whole 128-token tiles
        s = budget_blocks(1 - pct / 100, nK, 4)
        assert round(100 * (1 - s / nK), 2) == pct, (name, s, nK)


def test_workload_budgets_match_printed_sparsity():
    assert round(100 * (1 - WORKLOADS["wan14b"].s / WORKLOADS["wan14b"].nK), 2) == 89.16
    assert round(100 * (1 - WORKLOADS["wan13b"].s / WORKLOADS["wan13b"].nK), 2) == 89.16
    hy = WORKLOADS["hunyuan13b"]
    assert round(100 * (1 - hy.s / hy.nK), 2) == 92.35
    assert round(100 * hy.s / hy.nK, 2) == 7.65
