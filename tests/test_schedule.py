"""The denoising-loop schedule (dense first block and first 10 steps, plan rebuilt every 4
steps and reused in between): its decisions on the CPU, and on the GPU that every call it
makes equals the corresponding library call made by hand."""

import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv, perturb
from block_sparse_attention_ibcs_b200.schedule import (DENSE, REFRESH, REUSE, SparseAttentionSchedule,
                                                       refresh_index, schedule_mode)


def test_schedule_decisions():
    # 50 steps, 3 blocks: block 0 and steps 0..9 dense; then refresh at 10, 14, 18, ...
    for step in range(50):
        assert schedule_mode(0, step) == DENSE
        for block in (1, 2):
            m = schedule_mode(block, step)
            if step < 10:
                assert m == DENSE
            elif (step - 10) % 4 == 0:
                assert m == REFRESH and refresh_index(step) == (step - 10) // 4
            else:
                assert m == REUSE
    modes = [schedule_mode(1, t) for t in range(50)]
    assert modes.count(DENSE) == 10 and modes.count(REFRESH) == 10 and modes.count(REUSE) == 30
    assert [refresh_index(t) for t in (10, 13, 14, 49)] == [0, 0, 1, 9]
    assert schedule_mode(1, 4, dense_steps=3, refresh=2) == REUSE
    assert schedule_mode(1, 5, dense_steps=3, refresh=2) == REFRESH


@pytest.mark.gpu
def test_schedule_calls_equal_manual_library_calls():
    w = WORKLOADS["tiny"]
    Q0, K0, V0 = make_qkv(w, device="cuda")
    nblk, steps = 2, 17
    sch = SparseAttentionSchedule(w.B, w.H, w.N, w.d, nblk, w.s, seed=100)
    p = sch.p
    S = torch.empty_like(sch.S)
    ws = torch.empty_like(sch.ws)
    idx = torch.empty_like(sch.idx[1])
    lp = torch.empty_like(sch.logpi[1])
    for t in range(steps):
        Q, K, V = (perturb(x, 0.05, 1000 * t + k) for k, x in enumerate((Q0, K0, V0)))
        for b in range(nblk):
            O = torch.empty_like(Q)
            mode = sch.attention(b, t, Q, K, V, O)
            ref = torch.empty_like(Q)
            if mode == DENSE:
                ab.ab_attn_dense(p, Q, K, V, ref)
            else:
                if mode == REFRESH:  # the plan the schedule must have built
                    ab.ab_select(p, Q, K, S, ws)
                    ab.ab_plan(p, S, w.s, 100 + b, refresh_index(t), idx, lp)
                    assert torch.equal(idx, sch.idx[b]) and torch.equal(lp, sch.logpi[b])
                ab.ab_attn(p, Q, K, V, idx, lp, w.s, ref)
            assert ab.ab_get_status() == 0
            assert torch.equal(O, ref), (b, t, mode)
    assert sch.calls == {DENSE: steps + 10, REFRESH: 2, REUSE: 5}
