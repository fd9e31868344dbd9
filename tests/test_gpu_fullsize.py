"""Full-size parity: the workloads the bench runs, checked on sampled outputs.

Each stage runs on the whole tensor in the same launch configuration as bench.py; the
oracle recomputes a fixed sample of rows (first, last and interior query blocks of a
few heads).  Inputs come from the seeded generators only.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv, random_plan, random_scores
from oracle import abattn_oracle as O

from _util import assert_o_close, assert_s_close, f32_ulp_diff, np64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = ["wan13b", "wan14b", "hunyuan13b"]


def _sample_rows(w, k=3):
    rng = np.random.default_rng(w.seed)
    heads = sorted({0, w.H - 1} | set(rng.integers(0, w.H, 1).tolist()))
    rows = sorted({0, w.nQ - 1} | set(rng.integers(1, w.nQ - 1, k).tolist()))
    return heads, rows


@pytest.mark.parametrize("name", FULL)
def test_select_full_size(name):
    w = WORKLOADS[name]
    Q, K, _ = make_qkv(w, device="cuda")
    p = ab.params(w.B, w.H, w.N, w.d, w.kv_block)
    S = torch.empty(w.B, w.H, w.nQ, w.nK, device="cuda")
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    ab.ab_select(p, Q, K, S, ws)
    assert ab.ab_get_status() == 0
    # cheap invariant on every row: each S row sums to 1
    sums = S.double().sum(-1)
    assert (sums - 1).abs().max().item() < 1e-4
    heads, rows = _sample_rows(w)
    for h in heads[:2]:
        qh, kh = np64(Q[0, h]), np64(K[0, h])
        ref = O.select_head(qh, kh, 128, w.kv_block, 8, 1, rows=rows)
        got = S[0, h, rows].cpu().numpy()
        assert_s_close(got, ref, f"{name} h{h}")


@pytest.mark.parametrize("name", FULL)
def test_plan_full_size(name):
    w = WORKLOADS[name]
    R = w.B * w.H * w.nQ
    S = random_scores(R, w.nK, seed=w.seed + 5, device="cuda")
    p = ab.params(w.B, w.H, w.N, w.d, w.kv_block)
    idx = torch.empty(R, w.s, dtype=torch.int32, device="cuda")
    lp = torch.empty(R, w.s, device="cuda")
    ab.ab_plan(p, S, w.s, w.philox_seed, 3, idx, lp)
    assert ab.ab_get_status() == 0
    ii = idx.cpu().numpy()
    assert (np.diff(ii, axis=1) > 0).all() and ii.min() >= 0 and ii.max() < w.nK
    pick = [0, R - 1, R // 3, (2 * R) // 3, w.nQ - 1]
    S_cpu = S[torch.tensor(pick, device="cuda")].cpu().numpy()
    lpc = lp.cpu().numpy()
    for k, r in enumerate(pick):
        ridx, rlp, _ = O.plan_row(S_cpu[k], w.s, w.philox_seed, 3, r)
        assert np.array_equal(ii[r], ridx), f"{name} row {r}"
        assert f32_ulp_diff(lpc[r], rlp).max() <= 1


@pytest.mark.parametrize("name", FULL + ["sweep_bk16", "sweep_bk64", "sweep_bk128"])
def test_attn_full_size(name):
    w = WORKLOADS[name]
    Q, K, V = make_qkv(w, device="cuda")
    R = w.B * w.H * w.nQ
    idx, lp = random_plan(R, w.nK, w.s, seed=w.seed + 9, device="cuda")
    p = ab.params(w.B, w.H, w.N, w.d, w.kv_block)
    Od = torch.empty_like(Q)
    ab.ab_attn(p, Q, K, V, idx, lp, w.s, Od)
    assert ab.ab_get_status() == 0
    assert torch.isfinite(Od.float()).all()
    heads, rows = _sample_rows(w)
    for h in heads[:2]:
        qh, kh, vh = np64(Q[0, h]), np64(K[0, h]), np64(V[0, h])
        oh = Od[0, h]
        for i in rows:
            r = h * w.nQ + i
            ref = O.attn_block(qh[i * 128: min(w.N, (i + 1) * 128)], kh, vh,
                               idx[r].cpu().numpy(), lp[r].cpu().numpy(), w.kv_block)
            got = np64(oh[i * 128: min(w.N, (i + 1) * 128)])
            assert_o_close(got, ref, f"{name} h{h} qb{i}")


def test_all_blocks_packed_equals_dense_path_full_shape():
    """s = all blocks through the packed kernel == the dense path, Wan2.1-1.3B shape,
    bk = 128 (one block per tile), bitwise."""
    w = WORKLOADS["sweep_bk128"]
    Q, K, V = make_qkv(w, device="cuda", heads=[0, 1])
    H = 2
    p = ab.params(1, H, w.N, w.d, kv_block=128)
    nK = w.nK
    idx = torch.arange(nK, dtype=torch.int32, device="cuda").repeat(H * w.nQ, 1).contiguous()
    lp = torch.zeros(H * w.nQ, nK, device="cuda")
    O1 = torch.empty_like(Q)
    O2 = torch.empty_like(Q)
    ab.ab_attn(p, Q, K, V, idx, lp, nK, O1)
    ab.ab_attn_dense(p, Q, K, V, O2)
    assert ab.ab_get_status() == 0
    assert torch.equal(O1, O2)
    ref = O.dense_attention(np64(Q[0, 0, -80:]), np64(K[0, 0]), np64(V[0, 0]))
    assert_o_close(np64(O2[0, 0, -80:]), ref, "dense last query block")
