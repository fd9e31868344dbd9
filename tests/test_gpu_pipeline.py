"""The whole path (ab_select -> ab_plan -> ab_attn) on batches of several sequences and on
KV blocks of 1 and 2 tokens, each stage checked against the oracle on the GPU's own inputs:
S within 1e-4 relative (labels may differ only at oracle near-ties), plans bit-exact for the
GPU's S with Philox row = (b H + h) nQ + i, O within the attention tolerance."""

import numpy as np
import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import gaussian_head
from oracle import abattn_oracle as O

from _util import assert_o_close, assert_s_close, f32_ulp_diff, np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,d,bk,s", [
    (2, 3, 300, 64, 4, 20),     # batch of 2, ragged last query block (44 rows)
    (3, 1, 260, 128, 16, 5),    # batch of 3, d = 128, last KV block 4 tokens
    (2, 2, 256, 64, 2, 40),     # 2-token blocks: 64 blocks per tile
    (1, 2, 200, 64, 1, 70),     # 1-token blocks: 128 blocks per tile, ragged tile
])
def test_pipeline_batches_and_small_blocks(B, H, N, d, bk, s):
    seed = 1000 * B + 10 * H + bk
    def head(k, b, h):
        return gaussian_head(N, d, seed * 97 + 31 * (b * H + h) + k)
    Q = torch.stack([torch.stack([head(0, b, h) for h in range(H)]) for b in range(B)]).bfloat16()
    K = torch.stack([torch.stack([head(1, b, h) for h in range(H)]) for b in range(B)]).bfloat16()
    V = torch.stack([torch.stack([head(2, b, h) for h in range(H)]) for b in range(B)]).bfloat16()
    nQ, nK = -(-N // 128), -(-N // bk)
    p = ab.params(B, H, N, d, kv_block=bk)
    S = torch.full((B, H, nQ, nK), float("nan"), device="cuda")
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    labels = torch.full((B, H, nQ * 128), 99, dtype=torch.int8, device="cuda")
    Qc, Kc, Vc = Q.cuda(), K.cuda(), V.cuda()
    ab.ab_select_debug(p, Qc, Kc, S, ws, labels)
    rows = B * H * nQ
    idx = torch.full((rows, s), -1, dtype=torch.int32, device="cuda")
    lp = torch.full((rows, s), 9.0, device="cuda")
    seed_p, off = 77, 5
    ab.ab_plan(p, S, s, seed_p, off, idx, lp)
    Od = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    ab.ab_attn(p, Qc, Kc, Vc, idx, lp, s, Od)
    assert ab.ab_get_status() == 0
    S_c, lab = S.cpu().numpy(), labels.cpu().numpy()
    idx_c, lp_c = idx.cpu().numpy(), lp.cpu().numpy()
    for b in range(B):
        for h in range(H):
            Qh, Kh, Vh = np64(Q[b, h]), np64(K[b, h]), np64(V[b, h])
            Kp = O.pool_keys(Kh, bk)
            for i in range(nQ):
                sl = slice(i * 128, min(N, (i + 1) * 128))
                Qb = Qh[sl]
                cref, wref, lref, gap = O.kmeans_block(Qb, 8, 1)
                lg = lab[b, h, sl].astype(np.int64)
                diff = lg != lref
                assert (gap[diff] < 1e-12).all(), f"b{b} h{h} qb{i}: labels differ off a near-tie"
                Sref = (O.scores_from_labels(Qb, lg, Kp, 8) if diff.any()
                        else O.block_scores(cref, wref, Kp).astype(np.float32))
                assert_s_close(S_c[b, h, i], Sref, f"b{b} h{h} qb{i}")
                r = (b * H + h) * nQ + i
                ridx, rlp, _ = O.plan_row(S_c[b, h, i], s, seed_p, off, r)
                assert np.array_equal(idx_c[r], ridx), f"row {r}: plan differs"
                assert f32_ulp_diff(lp_c[r], rlp).max() <= 1
                ref = O.attn_block(Qb, Kh, Vh, idx_c[r], lp_c[r], bk)
                assert_o_close(np64(Od[b, h, sl]), ref, f"b{b} h{h} qb{i}")
