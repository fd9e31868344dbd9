"""GPU parity of the packed-tile attention (ab_attn, ab_attn_dense) against the fp64 oracle.

Tolerance on O (bf16 inputs, fp32 accumulation, bf16 output, identical plan):
max-abs <= 1e-2 and relative L2 <= 5e-3.
"""

import math

import numpy as np
import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, gaussian_head, make_qkv, random_plan
from oracle import abattn_oracle as O

from _util import assert_o_close, np64

pytestmark = pytest.mark.gpu


def _qkv(H, N, d, seed):
    Q = torch.stack([gaussian_head(N, d, seed * 100 + 3 * h) for h in range(H)])[None].bfloat16()
    K = torch.stack([gaussian_head(N, d, seed * 100 + 3 * h + 1) for h in range(H)])[None].bfloat16()
    V = torch.stack([gaussian_head(N, d, seed * 100 + 3 * h + 2) for h in range(H)])[None].bfloat16()
    return Q, K, V


def _run(p, Q, K, V, idx, lp, s):
    O_ = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    ab.ab_attn(p, Q.cuda(), K.cuda(), V.cuda(), idx.cuda(), lp.cuda(), s, O_)
    assert ab.ab_get_status() == 0
    return O_


def _check(O_gpu, Q, K, V, idx, lp, H, N, bk, qblocks=None):
    nQ = -(-N // 128)
    idx = idx.reshape(H, nQ, -1).numpy()
    lp = lp.reshape(H, nQ, -1).numpy()
    for h in range(H):
        Qh, Kh, Vh = np64(Q[0, h]), np64(K[0, h]), np64(V[0, h])
        Oh = np64(O_gpu[0, h])
        for i in (range(nQ) if qblocks is None else qblocks):
            rows = slice(i * 128, min(N, (i + 1) * 128))
            ref = O.attn_block(Qh[rows], Kh, Vh, idx[h, i], lp[h, i], bk)
            assert_o_close(Oh[rows], ref, f"h{h} qb{i}")


@pytest.mark.parametrize("N,d,bk,s", [
    (1024, 64, 4, 32),     # tiny config budget: one full tile
    (1024, 64, 4, 256),    # all blocks (8 tiles)
    (1000, 64, 4, 33),     # ragged query block (104 rows) + partial tile (132 tokens)
    (1000, 128, 16, 20),   # d = 128, partial last KV block handled by masking
    (1000, 64, 64, 9),     # last KV block has 40 valid tokens
    (1000, 128, 128, 5),   # one block per tile, last block 104 tokens
    (777, 64, 1, 300),     # single-token blocks, odd N
    (130, 128, 2, 65),     # two query blocks, the second with 2 rows
])
def test_attn_random_plan(N, d, bk, s):
    H = 2
    nQ, nK = -(-N // 128), -(-N // bk)
    Q, K, V = _qkv(H, N, d, seed=N + d + bk)
    idx, lp = random_plan(H * nQ, nK, s, seed=5)
    p = ab.params(1, H, N, d, kv_block=bk)
    O_ = _run(p, Q, K, V, idx, lp, s)
    _check(O_, Q, K, V, idx, lp, H, N, bk)


def test_attn_tiny_config_identical_oracle_plan():
    w = WORKLOADS["tiny"]
    Q, K, V = make_qkv(w)
    S = np.stack([O.select_head(np64(Q[0, h]), np64(K[0, h]), 128, 4, 8, 1) for h in range(w.H)])
    idx = np.zeros((w.H, w.nQ, w.s), np.int32)
    lp = np.zeros((w.H, w.nQ, w.s), np.float32)
    for h in range(w.H):
        for i in range(w.nQ):
            idx[h, i], lp[h, i], _ = O.plan_row(S[h, i], w.s, w.philox_seed, 0, h * w.nQ + i)
    idx_t, lp_t = torch.from_numpy(idx).reshape(-1, w.s), torch.from_numpy(lp).reshape(-1, w.s)
    p = ab.params(w.B, w.H, w.N, w.d, w.kv_block)
    O_ = _run(p, Q, K, V, idx_t, lp_t, w.s)
    _check(O_, Q, K, V, idx_t, lp_t, w.H, w.N, w.kv_block)


@pytest.mark.parametrize("N,d", [(1024, 64), (1000, 128), (300, 64)])
def test_dense_path_equals_dense_oracle(N, d):
    H = 2
    Q, K, V = _qkv(H, N, d, seed=7 + N)
    p = ab.params(1, H, N, d, kv_block=4)
    O_ = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    ab.ab_attn_dense(p, Q.cuda(), K.cuda(), V.cuda(), O_)
    assert ab.ab_get_status() == 0
    for h in range(H):
        ref = O.dense_attention(np64(Q[0, h]), np64(K[0, h]), np64(V[0, h]))
        assert_o_close(np64(O_[0, h]), ref, f"dense h{h}")


@pytest.mark.parametrize("bk", [4, 16, 128])
def test_all_blocks_packed_equals_dense_path_bitwise(bk):
    """s = nK gives pi = 1 (log pi = 0) and the packed tiles are exactly the dense tiles."""
    H, N, d = 2, 1024, 128
    nK = N // bk
    Q, K, V = _qkv(H, N, d, seed=3)
    p = ab.params(1, H, N, d, kv_block=bk)
    idx = torch.arange(nK, dtype=torch.int32).repeat(H * 8, 1)
    lp = torch.zeros(H * 8, nK)
    O1 = _run(p, Q, K, V, idx, lp, nK)
    O2 = torch.empty_like(O1)
    ab.ab_attn_dense(p, Q.cuda(), K.cuda(), V.cuda(), O2)
    assert ab.ab_get_status() == 0
    assert torch.equal(O1, O2)


@pytest.mark.parametrize("spike_nats", [38.0, 60.0])
def test_late_logit_spikes(spike_nats):
    """Logits far above the first tile's maximum in later tiles, for warp 0 of a query block.

    The softmax takes its exponentials against the running reference and falls back to
    the tile maximum (with a rescale of O) only when a tile's row sum passes 2^64.  With
    a spike of 38 nats (about 2^55 over the reference) every tile stays on the fast path
    with P values near 2^52; with 60 nats the tile holding it (tile 5) takes the fallback
    after an intermediate spike of 36 nats in tile 3 that does not.  Warps 1-3 of the
    block have no spike, so the fallback is exercised per warp."""
    H, N, d, bk = 1, 1024, 64, 4
    nK = N // bk
    Q, K, V = _qkv(H, N, d, seed=11)
    g = torch.Generator().manual_seed(7)
    u = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).float()  # |u|^2 = d
    beta = spike_nats * math.sqrt(d) / d  # (beta u) . u / sqrt(d) = spike_nats
    Q[0, 0, :32] = u.bfloat16()
    K[0, 0, 5 * 128 + 7] = (beta * u).bfloat16()
    K[0, 0, 3 * 128 + 9] = (0.6 * beta * u).bfloat16()
    p = ab.params(1, H, N, d, kv_block=bk)
    idx = torch.arange(nK, dtype=torch.int32).repeat(H * 8, 1)
    lp = torch.zeros(H * 8, nK)
    O_ = _run(p, Q, K, V, idx, lp, nK)
    _check(O_, Q, K, V, idx, lp, H, N, bk, qblocks=[0, 1])
    # the spike dominates warp 0's rows (the rest of the row's mass is below e^-20)
    assert np.abs(np64(O_[0, 0, :32]) - np64(V[0, 0, 5 * 128 + 7])).max() < 1e-2


def test_bad_index_status():
    H, N, d, bk, s = 1, 256, 64, 4, 8
    Q, K, V = _qkv(H, N, d, seed=9)
    idx = torch.arange(s, dtype=torch.int32).repeat(2, 1)
    idx[1, 3] = 10_000
    lp = torch.zeros(2, s)
    p = ab.params(1, H, N, d, kv_block=bk)
    O_ = torch.empty(Q.shape, dtype=torch.bfloat16, device="cuda")
    ab.ab_attn(p, Q.cuda(), K.cuda(), V.cuda(), idx.cuda(), lp.cuda(), s, O_)
    assert ab.ab_get_status() == -7
    assert ab.ab_get_status() == 0  # cleared
    # the masked block is simply absent: query block 1 attends to the 7 valid blocks
    keep = [0, 1, 2, 4, 5, 6, 7]
    ref = O.attn_block(np64(Q[0, 0, 128:]), np64(K[0, 0]), np64(V[0, 0]), keep, [0.0] * 7, bk)
    assert_o_close(np64(O_[0, 0, 128:]), ref)


def test_non_ascending_plan_rows_are_flagged():
    """Plan rows must be strictly ascending.  A duplicate (also across a tile edge) or an
    out-of-order block makes the validation pass record AB_ERR_DEVICE_CHECK; nothing
    faults, and the rows that keep the rules are attended as usual."""
    H, N, d, bk, s = 1, 1024, 64, 4, 64  # 32 blocks per tile: two tiles per row
    Q, K, V = _qkv(H, N, d, seed=17)
    nQ = N // 128
    good = (2 * torch.arange(s, dtype=torch.int32)).repeat(nQ, 1)  # 0, 2, ..., 126
    lp = -torch.rand(nQ, s, generator=torch.Generator().manual_seed(5)) * 2.0
    p = ab.params(1, H, N, d, kv_block=bk)
    O_ = torch.empty(Q.shape, dtype=torch.bfloat16, device="cuda")
    Qh, Kh, Vh = np64(Q[0, 0]), np64(K[0, 0]), np64(V[0, 0])
    bad_rows = {1: (32, None), 2: (10, 5), 3: (21, None), 6: (63, 0)}
    for row, (m, val) in bad_rows.items():
        idx = good.clone()
        # None: repeat the entry before (row 1: the first entry of tile 1 repeats the last
        # of tile 0; row 3: adjacent duplicate inside a tile); else an out-of-order value
        idx[row, m] = idx[row, m - 1] if val is None else val
        ab.ab_attn(p, Q.cuda(), K.cuda(), V.cuda(), idx.cuda(), lp.cuda(), s, O_)
        assert ab.ab_get_status() == -7, f"row {row}"
        assert ab.ab_get_status() == 0  # cleared
        for i in (0, 7):  # rows that keep the rules
            ref = O.attn_block(Qh[i * 128:(i + 1) * 128], Kh, Vh, good[i].numpy(), lp[i].numpy(), bk)
            assert_o_close(np64(O_[0, 0, i * 128:(i + 1) * 128]), ref, f"qb{i}")
    # a valid plan leaves the status word clear
    ab.ab_attn(p, Q.cuda(), K.cuda(), V.cuda(), good.cuda(), lp.cuda(), s, O_)
    assert ab.ab_get_status() == 0


@pytest.mark.parametrize("s,m", [(256, 128), (256, 255), (33, 17), (33, 32)])
def test_plan_validation_across_steps_and_odd_budgets(s, m):
    """The validation pass reads four entries per lane (a 128-entry step per warp) when the
    rows are 16-byte aligned, one per lane otherwise: a repeated entry is found at a step
    boundary, at the row's end, and with an odd budget s."""
    H, N, d, bk = 1, 1024, 64, 4
    Q, K, V = _qkv(H, N, d, seed=19)
    nQ, nK = N // 128, N // bk
    rng = np.random.default_rng(s + m)
    good = torch.from_numpy(np.stack([np.sort(rng.choice(nK, s, replace=False))
                                      for _ in range(nQ)]).astype(np.int32))
    lp = torch.zeros(nQ, s)
    p = ab.params(1, H, N, d, kv_block=bk)
    O_ = torch.empty(Q.shape, dtype=torch.bfloat16, device="cuda")
    ab.ab_attn(p, Q.cuda(), K.cuda(), V.cuda(), good.cuda(), lp.cuda(), s, O_)
    assert ab.ab_get_status() == 0
    bad = good.clone()
    bad[5, m] = bad[5, m - 1]
    ab.ab_attn(p, Q.cuda(), K.cuda(), V.cuda(), bad.cuda(), lp.cuda(), s, O_)
    assert ab.ab_get_status() == -7


def test_device_wait_timeout_is_reported_and_context_survives():
    """A producer that never signals tile 0: the bounded waits give up after 50 ms, the
    status word reports AB_ERR_DEVICE_TIMEOUT, and the context stays usable."""
    H, N, d, bk, s = 1, 256, 64, 4, 64
    Q, K, V = _qkv(H, N, d, seed=13)
    idx, lp = random_plan(2, N // bk, s, seed=1)
    p = ab.params(1, H, N, d, kv_block=bk)
    O_ = torch.empty(Q.shape, dtype=torch.bfloat16, device="cuda")
    args = (p, Q.cuda(), K.cuda(), V.cuda(), idx.cuda(), lp.cuda(), s, O_)
    ab.ab_attn_debug(*args, 1, 50_000_000)
    assert ab.ab_get_status() == -4
    # the same call without the skipped arrival works afterwards
    ab.ab_attn_debug(*args, 0, 2_000_000_000)
    assert ab.ab_get_status() == 0
    _check(O_.cpu(), Q, K, V, idx, lp, H, N, bk)


def test_traced_kernel_matches_and_orders_its_events():
    """The traced kernel (ab_attn_debug with a trace buffer) gives the untraced O bit for bit,
    and each traced tile's events keep the orders that program order and the pipeline's
    barriers guarantee: a tile's copies start before they are issued and before its K or V
    can land; QK is issued after K landed, S is seen after that, and the softmax loads S and
    builds P after seeing it; PV is issued after V landed and after S was seen."""
    H, N, d, bk, s = 2, 8192, 128, 4, 512  # 64 query blocks, 16 tiles each
    Q, K, V = _qkv(H, N, d, seed=21)
    nQ = N // 128
    idx, lp = random_plan(H * nQ, N // bk, s, seed=4)
    p = ab.params(1, H, N, d, kv_block=bk)
    O_ref = _run(p, Q, K, V, idx, lp, s)
    O_tr = torch.empty_like(O_ref)
    tr = torch.zeros(3 * 16 * 128, dtype=torch.int64, device="cuda")
    ab.ab_attn_debug(p, Q.cuda(), K.cuda(), V.cuda(), idx.cuda(), lp.cuda(), s, O_tr, 0, 2_000_000_000, tr)
    assert ab.ab_get_status() == 0
    assert torch.equal(O_tr, O_ref)
    ev = tr.view(3, 16, 128).cpu().numpy()
    T = s * bk // 128
    for slot in range(3):
        e = ev[slot][:, :T]
        assert (e[[0, 1, 2, 3, 4, 5, 7, 8, 9, 10, 12, 13, 14, 15]] > 0).all(), f"slot {slot}: missing events"
        assert (e[1] >= e[0]).all() and (e[4] >= e[0]).all() and (e[12] >= e[0]).all()
        assert (e[5] >= e[4]).all() and (e[9] >= e[4]).all()
        assert (e[2] >= e[9]).all() and (e[3] >= e[2]).all()
        assert (e[7] >= e[12]).all() and (e[7] >= e[9]).all()
