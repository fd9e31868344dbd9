"""GPU parity of the SIP planner (ab_plan, ab_sample) against the CPU oracle.

Sample indices must be bit-exact; log-probabilities may differ by at most one fp32
ulp (the fp64 logarithm is rounded to fp32 on both sides, and CUDA's and the host's
fp64 log may differ in the last fp64 bit).
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv, random_scores
from oracle import abattn_oracle as O

from _util import f32_ulp_diff, np64

pytestmark = pytest.mark.gpu

TWO32 = 1 << 32


def _gpu_plan(p, S, s, seed, offset, fn=ab.ab_plan):
    rows = S.shape[0] * S.shape[1] * S.shape[2] if S.dim() == 4 else S.shape[0]
    idx = torch.full((rows, s), -7, dtype=torch.int32, device="cuda")
    lp = torch.full((rows, s), 99.0, dtype=torch.float32, device="cuda")
    fn(p, S.contiguous(), s, seed, offset, idx, lp)
    assert ab.ab_get_status() == 0
    return idx.cpu().numpy(), lp.cpu().numpy()


def _check_rows(S_cpu, idx, lp, s, seed, offset, rows):
    for r in rows:
        ridx, rlp, qp = O.plan_row(S_cpu[r], s, seed, offset, r)
        assert np.array_equal(idx[r], ridx), f"row {r}: idx differs"
        assert f32_ulp_diff(lp[r], rlp).max() <= 1, f"row {r}: logpi differs"
        assert int(qp.sum()) == s * TWO32


def test_plan_tiny_config_from_oracle_scores():
    w = WORKLOADS["tiny"]
    Q, K, _ = make_qkv(w)
    S = np.stack([O.select_head(np64(Q[0, h]), np64(K[0, h]), 128, w.kv_block, 8, 1)
                  for h in range(w.H)])  # [H, nQ, nK] fp32
    p = ab.params(w.B, w.H, w.N, w.d, w.kv_block)
    St = torch.from_numpy(S).cuda().reshape(1, w.H, w.nQ, w.nK)
    for s in (32, 1, 255, 256):
        idx, lp = _gpu_plan(p, St, s, w.philox_seed, 0)
        _check_rows(S.reshape(-1, w.nK), idx, lp, s, w.philox_seed, 0, range(w.H * w.nQ))
    # s = all blocks: pi = 1 everywhere
    idx, lp = _gpu_plan(p, St, 256, 5, 3)
    assert (idx == np.arange(256)).all() and (lp == 0).all()


@pytest.mark.parametrize("name", ["wan13b", "hunyuan13b"])
def test_plan_full_shape_random_scores(name):
    w = WORKLOADS[name]
    rows = w.B * w.H * w.nQ
    S = random_scores(rows, w.nK, seed=11, device="cuda")
    p = ab.params(w.B, w.H, w.N, w.d, w.kv_block)
    idx, lp = _gpu_plan(p, S, w.s, w.philox_seed, 7)
    # every row: exactly s distinct ascending in-range indices (cheap host invariants)
    assert (np.diff(idx, axis=1) > 0).all() and idx.min() >= 0 and idx.max() < w.nK
    assert (lp <= 0).all()
    pick = [0, 1, w.nQ - 1, rows // 2, rows - 1] + list(np.random.default_rng(0).integers(0, rows, 11))
    S_cpu = S[torch.tensor(pick, device="cuda")].cpu().numpy()
    for k, r in enumerate(pick):
        ridx, rlp, _ = O.plan_row(S_cpu[k], w.s, w.philox_seed, 7, int(r))
        assert np.array_equal(idx[r], ridx), f"row {r}"
        assert f32_ulp_diff(lp[r], rlp).max() <= 1


def test_plan_edge_rows():
    nK = 256
    rows = []
    rng = np.random.default_rng(3)
    x = np.exp(2 * rng.standard_normal(nK)); rows.append(x / x.sum())        # ordinary
    z = np.zeros(nK); z[[5, 9, 200]] = [0.5, 0.3, 0.2]; rows.append(z)        # fewer than s positive
    o = np.full(nK, 1e-9); o[17] = 1.0; rows.append(o / o.sum())              # one dominant block
    u = np.full(nK, 1.0 / nK); rows.append(u)                                 # uniform
    t = np.exp(6 * rng.standard_normal(nK)); rows.append(t / t.sum())         # very heavy tail
    n = x / x.sum(); n = n.copy(); n[[3, 4]] = np.nan; n[7] = -1.0; rows.append(n)  # NaN / negative
    e = np.zeros(nK); rows.append(e)                                          # all zero
    d = np.exp(rng.standard_normal(nK)); d[100:] = 0; rows.append(d / d.sum())  # zero tail
    S = np.stack(rows).astype(np.float32)
    R = len(rows)
    assert R == 8  # N = 1024 tokens: 8 query blocks x 256 KV blocks of 4
    p = ab.params(1, 1, 1024, 64, kv_block=4)
    for s in (1, 8, 32, 255):
        idx, lp = _gpu_plan(p, torch.from_numpy(S).cuda(), s, 123, 456)
        _check_rows(S, idx, lp, s, 123, 456, range(R))


def test_sample_given_oracle_pi_bit_exact():
    rng = np.random.default_rng(4)
    nK, R, s = 256, 8, 24
    S = rng.dirichlet(np.full(nK, 0.3), size=R).astype(np.float32)
    pi = np.stack([(O.inclusion_fixed_point(S[r], s)[0].astype(np.float64) / TWO32) for r in range(R)])
    pi = pi.astype(np.float32)
    p = ab.params(1, 1, 128 * R, 64, kv_block=4)
    assert -(-128 * R // 4) == nK
    idx, lp = _gpu_plan(p, torch.from_numpy(pi).cuda(), s, 9, 1, fn=ab.ab_sample)
    for r in range(R):
        ridx, rlp, qp = O.sample_row(pi[r], s, 9, 1, r)
        assert np.array_equal(idx[r], ridx)
        assert f32_ulp_diff(lp[r], rlp).max() <= 1
        # the draw reproduces the given probabilities to fp32 resolution (the fixed-point
        # cap may move about s * 2^-23 of mass off the last non-saturated block)
        assert np.allclose(qp.astype(np.float64) / TWO32, pi[r], rtol=2e-6, atol=s * 2.0 ** -22)


def test_sample_monte_carlo_inclusion_frequencies():
    """Over many offsets the GPU's inclusion frequencies match pi (same rows, new U)."""
    rng = np.random.default_rng(5)
    nK, s = 256, 20
    x = np.exp(1.5 * rng.standard_normal(nK))
    S = (x / x.sum()).astype(np.float32)
    R = 2048  # rows = independent draws (the row index enters the Philox counter)
    p = ab.params(1, R // 8, 1024, 64, kv_block=4)  # 256 heads x 8 query blocks, nK = 256
    St = torch.from_numpy(np.tile(S, (R, 1))).cuda()
    idx, _ = _gpu_plan(p, St, s, 77, 0)
    hits = np.bincount(idx.ravel(), minlength=nK) / R
    qp, _, _ = O.inclusion_fixed_point(S, s)
    pi = qp.astype(np.float64) / TWO32
    se = np.sqrt(np.maximum(pi * (1 - pi), 1e-12) / R)
    assert np.abs((hits - pi) / se)[(pi > 0) & (pi < 1)].max() < 5.5
    assert (hits[pi == 1] == 1).all()


def test_plan_stress_rows_every_path():
    """Many varied rows, every one bit-exact.  Of the 8,000 (row, s) cases the planner's
    search brackets lambda* in its single three-candidate pass for 3,837, after the Newton
    step for 447, after doubling and bisection for 2,708, and 1,008 have fewer positive
    scores than s (counted by a CPU emulation of the search).  The step down from below the
    three candidates needs every product at lambda0's lower neighbour rounded up by the
    full 2^-24, which these rows never reach."""
    rng = np.random.default_rng(12)
    nK, R = 256, 2000
    rows = []
    for r in range(R):
        kind = r % 8
        if kind == 0:
            x = rng.dirichlet(np.full(nK, 0.05))                           # very peaked
        elif kind == 1:
            x = np.exp(rng.uniform(0.5, 8.0) * rng.standard_normal(nK))    # heavy tails
        elif kind == 2:
            x = rng.dirichlet(np.full(nK, 1.0)) * 10.0 ** rng.uniform(-6, 6)  # unnormalised
        elif kind == 3:
            x = np.full(nK, 1.0 / nK) * (1 + 1e-7 * rng.standard_normal(nK))  # near ties
        elif kind == 4:
            x = rng.dirichlet(np.full(nK, 0.3)); x[rng.random(nK) < 0.7] = 0.0  # many zeros
        elif kind == 5:
            x = np.zeros(nK); x[rng.integers(0, nK, 3)] = rng.random(3) + 0.1   # few positive
        elif kind == 6:
            x = rng.dirichlet(np.full(nK, 0.5)); x[rng.integers(0, nK, 2)] = np.nan
            x[rng.integers(0, nK, 2)] = -1.0                                 # NaN / negative
        else:
            x = rng.random(nK) ** 12                                         # skewed uniform
        rows.append(x)
    S = np.stack(rows).astype(np.float32)
    # one launch covers B*H*nQ rows: R/8 heads of 8 query blocks (N = 1024, nK = 256)
    p = ab.params(1, R // 8, 1024, 64, kv_block=4)
    St = torch.from_numpy(S).cuda().reshape(1, R // 8, 8, nK)
    for s in (1, 7, 64, 200):
        idx, lp = _gpu_plan(p, St, s, 77, 5)
        _check_rows(S, idx, lp, s, 77, 5, range(R))


@pytest.mark.parametrize("nK", [18_940, 18_941, 18_944, 28_677, 29_700])
def test_plan_rows_at_the_staging_limit(nK):
    """Rows of exactly the planner's staging size (18,940 scores, the whole row in shared
    memory) and past it (the first 18,940 staged, the tail re-read from global memory on
    every pass), with nK a multiple of 4 (one bulk copy; 16-byte tail loads) and odd
    (strided staging; scalar tail loads), up to a HunyuanVideo-length row: every path draws
    the oracle's plan.  A stress mix of rows: heavy tails, a saturated block, zeros, NaN."""
    rng = np.random.default_rng(nK)
    N = 4 * nK  # KV blocks of 4 tokens
    nQ = -(-N // 128)
    R = 6  # rows checked; the launch covers all nQ rows of one head
    S = torch.from_numpy(np.abs(rng.standard_normal((nQ, nK))).astype(np.float32) ** 3)
    rows = []
    x = np.exp(3 * rng.standard_normal(nK)); rows.append(x / x.sum())
    y = np.full(nK, 1e-6); y[nK - 2] = 0.5; rows.append(y / y.sum())      # saturated in the tail
    z = rng.random(nK); z[: nK // 2] = 0.0; rows.append(z)                  # zeros up front
    t = rng.random(nK) ** 9; t[nK - 1] = np.nan; rows.append(t)             # NaN at the end
    u = np.full(nK, 1.0); rows.append(u)                                    # flat
    v = rng.dirichlet(np.full(nK, 0.2)); rows.append(v)
    S[:R] = torch.from_numpy(np.stack(rows).astype(np.float32))
    p = ab.params(1, 1, N, 64, kv_block=4)
    for s in (64, 2048):
        idx, lp = _gpu_plan(p, S.cuda().reshape(1, 1, nQ, nK), s, 31, 2)
        _check_rows(S.numpy(), idx, lp, s, 31, 2, list(range(R)) + [nQ - 1])
