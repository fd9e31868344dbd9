"""GPU parity of the IBCS selector (ab_select / ab_select_debug) against the CPU oracle.

Pooled keys and centroids must match bit for bit (both sides round exact fp64 means
once to bf16), shares exactly, cluster labels exactly except where the oracle's
best/second-best distance gap is below 1e-12 relative (fp64 summation order decides
such near-ties; those query blocks are re-scored with the GPU's labels), and S within
1e-4 relative per element.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, gaussian_head, make_qkv
from oracle import abattn_oracle as O

from _util import assert_s_close, np64

pytestmark = pytest.mark.gpu

NEAR_TIE = 1e-12


def _select_gpu(p, Q, K, C, nQ, nK, N, d, H):
    S = torch.full((1, H, nQ, nK), float("nan"), device="cuda")
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    labels = torch.full((1, H, nQ * 128), 99, dtype=torch.int8, device="cuda")
    cent = torch.empty((1, H, nQ, C, d), dtype=torch.bfloat16, device="cuda")
    w = torch.empty((1, H, nQ, C), device="cuda")
    Kp = torch.empty((1, H, nK, d), dtype=torch.bfloat16, device="cuda")
    ab.ab_select_debug(p, Q.cuda(), K.cuda(), S, ws, labels, cent, w, Kp)
    assert ab.ab_get_status() == 0
    return S.cpu().numpy(), labels.cpu().numpy(), np64(cent), w.cpu().numpy(), np64(Kp)


def _compare_head(Qh, Kh, h, bk, C, iters, S, labels, cent, w, Kp, rows=None):
    N = Qh.shape[0]
    nQ = -(-N // 128)
    Kp_ref = O.pool_keys(Kh, bk)
    assert np.array_equal(Kp[0, h], Kp_ref), "pooled keys differ"
    for i in (range(nQ) if rows is None else rows):
        Qb = Qh[i * 128: min(N, (i + 1) * 128)]
        n = Qb.shape[0]
        cref, wref, lref, gap = O.kmeans_block(Qb, C, iters)
        lg = labels[0, h, i * 128: i * 128 + n].astype(np.int64)
        assert (labels[0, h, i * 128 + n: (i + 1) * 128] == -1).all()
        diff = lg != lref
        if diff.any():
            assert (gap[diff] < NEAR_TIE).all(), f"h{h} qb{i}: label mismatch off a near-tie"
            Sref = O.scores_from_labels(Qb, lg, Kp_ref, C)
        else:
            assert np.array_equal(cent[0, h, i], cref), f"h{h} qb{i}: centroids differ"
            assert np.array_equal(w[0, h, i].astype(np.float64), wref.astype(np.float32).astype(np.float64))
            Sref = O.block_scores(cref, wref, Kp_ref).astype(np.float32)
        assert_s_close(S[0, h, i], Sref, f"h{h} qb{i}")
        assert abs(S[0, h, i].astype(np.float64).sum() - 1) < 1e-4


@pytest.mark.parametrize("N,d,bk,C,iters", [
    (1024, 64, 4, 8, 1),    # tiny config shape
    (1000, 64, 4, 8, 1),    # ragged last query block (104 rows)
    (1000, 128, 64, 8, 1),  # last KV block of 40 tokens
    (1000, 64, 128, 5, 1),  # 5 clusters, 8 KV blocks
    (1024, 64, 16, 8, 0),   # segment means only (ablation)
    (1024, 64, 4, 8, 2),    # two Lloyd iterations
    (133, 128, 4, 8, 1),    # second query block has 5 rows (3 empty segments)
])
def test_select_gaussian(N, d, bk, C, iters):
    H = 2
    Q = torch.stack([gaussian_head(N, d, 11 + h) for h in range(H)])[None].bfloat16()
    K = torch.stack([gaussian_head(N, d, 21 + h) for h in range(H)])[None].bfloat16()
    nQ, nK = -(-N // 128), -(-N // bk)
    p = ab.params(1, H, N, d, kv_block=bk, clusters=C, kmeans_iters=iters)
    S, labels, cent, w, Kp = _select_gpu(p, Q, K, C, nQ, nK, N, d, H)
    for h in range(H):
        _compare_head(np64(Q[0, h]), np64(K[0, h]), h, bk, C, iters, S, labels, cent, w, Kp)


def test_select_tiny_config():
    wl = WORKLOADS["tiny"]
    Q, K, _ = make_qkv(wl)
    p = ab.params(wl.B, wl.H, wl.N, wl.d, wl.kv_block)
    S, labels, cent, w, Kp = _select_gpu(p, Q, K, 8, wl.nQ, wl.nK, wl.N, wl.d, wl.H)
    for h in range(wl.H):
        _compare_head(np64(Q[0, h]), np64(K[0, h]), h, 4, 8, 1, S, labels, cent, w, Kp)


def test_select_plain_entry_matches_debug_entry():
    wl = WORKLOADS["tiny"]
    Q, K, _ = make_qkv(wl)
    p = ab.params(wl.B, wl.H, wl.N, wl.d, wl.kv_block)
    S1 = torch.empty((1, wl.H, wl.nQ, wl.nK), device="cuda")
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    ab.ab_select(p, Q.cuda(), K.cuda(), S1, ws)
    S2, *_ = _select_gpu(p, Q, K, 8, wl.nQ, wl.nK, wl.N, wl.d, wl.H)
    assert ab.ab_get_status() == 0
    assert np.array_equal(S1.cpu().numpy(), S2)


def test_select_fourier_structured_small():
    """The structured generator (shared Fourier features) on a small latent."""
    from block_sparse_attention_ibcs_b200.inputs import Workload

    wl = Workload("small", 1, 2, (4, 12, 20), 128, 4, 64, "fourier", 5, 5)
    Q, K, _ = make_qkv(wl)
    p = ab.params(1, wl.H, wl.N, wl.d, 4)
    S, labels, cent, w, Kp = _select_gpu(p, Q, K, 8, wl.nQ, wl.nK, wl.N, wl.d, wl.H)
    for h in range(wl.H):
        _compare_head(np64(Q[0, h]), np64(K[0, h]), h, 4, 8, 1, S, labels, cent, w, Kp)
