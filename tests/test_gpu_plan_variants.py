"""GPU parity of the planner variants (ab_plan_variant) against the CPU oracle.

Top-k and the no-IPW / uniform variants of the SIP planner (AB-Attention page,
ablations).  Block indices must be bit-exact; log-probabilities are exactly 0 for
top-k and no-IPW and within one fp32 ulp of the oracle's for the sampled variants.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, random_scores
from oracle import abattn_oracle as O

from _util import f32_ulp_diff

pytestmark = pytest.mark.gpu

MODES = ["sip", "sip_no_ipw", "uniform", "topk"]


def _run(p, S, s, seed, offset, mode):
    rows = S.shape[0]
    idx = torch.full((rows, s), -7, dtype=torch.int32, device="cuda")
    lp = torch.full((rows, s), 99.0, dtype=torch.float32, device="cuda")
    ab.ab_plan_variant(p, S.contiguous(), s, seed, offset, mode, idx, lp)
    assert ab.ab_get_status() == 0
    return idx.cpu().numpy(), lp.cpu().numpy()


def _check(S_cpu, idx, lp, s, seed, offset, mode, rows):
    for r in rows:
        ridx, rlp = O.plan_row_variant(S_cpu[r], s, seed, offset, r, mode)
        assert np.array_equal(idx[r], ridx), f"{mode} row {r}: idx differs"
        if mode in ("topk", "sip_no_ipw"):
            assert (lp[r] == 0).all()
        else:
            assert f32_ulp_diff(lp[r], rlp).max() <= 1, f"{mode} row {r}: logpi differs"


def _params(nK, bk=4):
    # one head of N = nK * bk tokens: the planner reads S as [ceil(N/128), nK] rows
    return ab.params(1, 1, nK * bk, 64, kv_block=bk)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("nK,s", [(256, 32), (257, 1), (300, 300), (1000, 123)])
def test_variants_random_rows(mode, nK, s):
    p = _params(nK)
    nQ = (nK * 4 + 127) // 128
    S = random_scores(nQ, nK, seed=nK + s, device="cuda")
    idx, lp = _run(p, S, s, 5, 3, mode)
    _check(S.cpu().numpy(), idx, lp, s, 5, 3, mode, range(nQ))


@pytest.mark.parametrize("mode", MODES)
def test_variants_ties_and_zeros(mode):
    nK, s = 512, 64
    p = _params(nK)
    nQ = (nK * 4 + 127) // 128
    g = torch.Generator().manual_seed(9)
    S = (torch.randint(0, 5, (nQ, nK), generator=g).float() / 4.0)  # many exact ties, zeros
    S[1] = 0.0                          # all zero: the budget is unreachable
    S[2, : s // 2] = 1.0                # fewer than s positive blocks
    S[2, s // 2:] = 0.0
    S[3] = -0.0                         # negative zeros
    idx, lp = _run(p, S.cuda(), s, 1, 0, mode)
    _check(S.numpy(), idx, lp, s, 1, 0, mode, range(nQ))


@pytest.mark.parametrize("mode", ["topk", "uniform"])
def test_variants_full_row_length(mode):
    # Wan2.1-1.3B row length (nK = 18,900, s = 2048), a few rows
    w = WORKLOADS["wan13b"]
    p = _params(w.nK)
    nQ = (w.nK * 4 + 127) // 128  # the launch plans every one of these rows
    S = random_scores(nQ, w.nK, seed=w.seed + 17, device="cuda")
    idx, lp = _run(p, S, w.s, w.philox_seed, 2, mode)
    _check(S.cpu().numpy(), idx, lp, w.s, w.philox_seed, 2, mode, [0, 1, nQ // 2, nQ - 1])


def test_no_ipw_equals_sip_draw_on_gpu():
    nK, s = 1000, 100
    p = _params(nK)
    nQ = (nK * 4 + 127) // 128
    S = random_scores(nQ, nK, seed=4, device="cuda")
    a = _run(p, S, s, 2, 0, "sip")
    b = _run(p, S, s, 2, 0, "sip_no_ipw")
    assert np.array_equal(a[0], b[0]) and (b[1] == 0).all()
    c_idx = torch.empty(nQ, s, dtype=torch.int32, device="cuda")
    c_lp = torch.empty(nQ, s, device="cuda")
    ab.ab_plan(p, S, s, 2, 0, c_idx, c_lp)
    assert ab.ab_get_status() == 0
    assert np.array_equal(a[0], c_idx.cpu().numpy()) and np.array_equal(a[1], c_lp.cpu().numpy())
