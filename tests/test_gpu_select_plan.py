"""ab_select_plan (select then plan, overlapped across head groups on two streams) gives
bit-identical S, idx and log pi to ab_select followed by ab_plan."""

import numpy as np
import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


def _separate(p, Q, K, s, seed, off, S_shape, rows):
    S = torch.empty(S_shape, device="cuda")
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    ab.ab_select(p, Q, K, S, ws)
    idx = torch.empty(rows, s, dtype=torch.int32, device="cuda")
    lp = torch.empty(rows, s, device="cuda")
    ab.ab_plan(p, S, s, seed, off, idx, lp)
    assert ab.ab_get_status() == 0
    return S, idx, lp


@pytest.mark.parametrize("name,heads,groups,two", [
    ("tiny", None, 2, True), ("tiny", None, 0, True), ("tiny", None, 5, False),
    ("wan13b", [0, 1, 2, 3, 4], 3, True), ("wan13b", [0, 1, 2, 3, 4], 99, True),
    ("hunyuan13b", [0, 1, 2], 2, True),  # rows longer than the planner's staged prefix
])
def test_select_plan_equals_separate_calls(name, heads, groups, two):
    w = WORKLOADS[name]
    Q, K, _ = make_qkv(w, device="cuda", heads=heads)
    H = Q.shape[1]
    p = ab.params(w.B, H, w.N, w.d, w.kv_block)
    rows = w.B * H * w.nQ
    S_shape = (w.B, H, w.nQ, w.nK)
    S0, idx0, lp0 = _separate(p, Q, K, w.s, w.philox_seed, 3, S_shape, rows)
    S = torch.full(S_shape, -1.0, device="cuda")
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    idx = torch.full((rows, w.s), -1, dtype=torch.int32, device="cuda")
    lp = torch.full((rows, w.s), 9.0, device="cuda")
    s2 = torch.cuda.Stream() if two else None
    ab.ab_select_plan(p, Q, K, S, ws, w.s, w.philox_seed, 3, idx, lp, groups=groups, stream2=s2)
    assert ab.ab_get_status() == 0
    assert torch.equal(S, S0)
    assert torch.equal(idx, idx0)
    assert torch.equal(lp, lp0)
