"""Head sharding: a call over heads [head0, head0 + H) of a layer (ab_params.head0 and
heads_total) gives S, idx, log pi and O bitwise equal to the matching rows of one call
over the whole layer.  This is what lets each GPU of a head-parallel group process its own
heads with no exchange: the planner draws with the whole layer's Philox row numbers and the
selector rounds S as the whole layer would."""

import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import Workload, make_qkv

import bench

pytestmark = pytest.mark.gpu

# B = 2 (the row numbering crosses batch entries), N = 8100: 64 query blocks (the last of
# 36 rows), 2025 KV blocks (ragged last score tile).  The score passes cut each 32-query-
# block group's keys into 4 chunks for all 16 heads, but would choose 8 chunks for a 2-head
# slice on its own: the slice must follow the whole layer's choice.
W = Workload("slices", 2, 8, (1, 81, 100), 128, 4, 256, "fourier", 11, 12)


def _stage(p, Q, K, V, S_shape, rows, offset=5):
    S = torch.full(S_shape, -1.0, device="cuda")
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    ab.ab_select(p, Q, K, S, ws)
    idx = torch.full((rows, W.s), -1, dtype=torch.int32, device="cuda")
    lp = torch.full((rows, W.s), 9.0, device="cuda")
    ab.ab_plan(p, S, W.s, W.philox_seed, offset, idx, lp)
    O_ = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    ab.ab_attn(p, Q, K, V, idx, lp, W.s, O_)
    assert ab.ab_get_status() == 0
    return S, idx, lp, O_


def test_head_slices_equal_the_whole_layer_bitwise():
    Q, K, V = make_qkv(W, device="cuda")
    B, H, nQ, nK = W.B, W.H, W.nQ, W.nK
    p = ab.params(B, H, W.N, W.d, W.kv_block)
    S, idx, lp, O_ = _stage(p, Q, K, V, (B, H, nQ, nK), B * H * nQ)
    idx = idx.reshape(B, H, nQ, W.s)
    lp = lp.reshape(B, H, nQ, W.s)
    for r in range(3):  # heads 0-2, 3-5, 6-7
        h0, h1 = bench.shard_heads(H, 3, r)
        n = h1 - h0
        sl = [x[:, h0:h1].contiguous() for x in (Q, K, V)]
        ps = ab.params(B, n, W.N, W.d, W.kv_block, head0=h0, heads_total=H)
        S2, idx2, lp2, O2 = _stage(ps, *sl, (B, n, nQ, nK), B * n * nQ)
        assert torch.equal(S2, S[:, h0:h1]), f"S of heads {h0}-{h1}"
        assert torch.equal(idx2.reshape(B, n, nQ, W.s), idx[:, h0:h1]), f"idx of heads {h0}-{h1}"
        assert torch.equal(lp2.reshape(B, n, nQ, W.s), lp[:, h0:h1]), f"log pi of heads {h0}-{h1}"
        assert torch.equal(O2, O_[:, h0:h1]), f"O of heads {h0}-{h1}"
        # ab_select_plan (two streams, slices of the slice) agrees as well
        S3 = torch.full_like(S2, -1.0)
        ws = torch.empty(ab.ab_workspace_bytes(ps), dtype=torch.uint8, device="cuda")
        idx3 = torch.full_like(idx2, -1)
        lp3 = torch.full_like(lp2, 9.0)
        ab.ab_select_plan(ps, sl[0], sl[1], S3, ws, W.s, W.philox_seed, 5, idx3, lp3, groups=2,
                          stream2=torch.cuda.Stream())
        assert ab.ab_get_status() == 0
        assert torch.equal(S3, S2) and torch.equal(idx3, idx2) and torch.equal(lp3, lp2)


def test_a_slice_taken_as_a_whole_layer_draws_differently():
    # the same heads called without head0/heads_total number their plan rows from 0 and
    # choose their own score split: the result is a valid plan, but not the layer's
    Q, K, V = make_qkv(W, device="cuda", heads=[6, 7])
    B, n, nQ, nK = W.B, 2, W.nQ, W.nK
    own = _stage(ab.params(B, n, W.N, W.d, W.kv_block), Q, K, V, (B, n, nQ, nK), B * n * nQ)
    sliced = _stage(ab.params(B, n, W.N, W.d, W.kv_block, head0=6, heads_total=8), Q, K, V,
                    (B, n, nQ, nK), B * n * nQ)
    assert not torch.equal(own[1], sliced[1])
    assert not torch.equal(own[0], sliced[0])
