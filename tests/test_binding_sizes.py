"""The Python binding refuses buffers smaller than the call reads or writes (CPU, no GPU).

The size checks come before the device checks, so CPU tensors exercise them: a buffer one
element short raises, a buffer of the right size passes on to the next check ("must be a
CUDA tensor").
"""

import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab

B, H, N, d, bk, s = 1, 2, 1000, 64, 4, 32
nQ, nK = 8, 250


def _t(n, dtype=torch.float32):
    return torch.zeros(n, dtype=dtype)


def _qkv(short=None):
    n = B * H * N * d
    return {k: _t(n - (k == short), torch.bfloat16) for k in ("Q", "K", "V", "O")}


P = ab.params(B, H, N, d, kv_block=bk)
WS = _t(16, torch.uint8)


def test_select_sizes():
    t = _qkv("K")
    with pytest.raises(ValueError, match="K holds"):
        ab.ab_select(P, t["Q"], t["K"], _t(B * H * nQ * nK), WS)
    t = _qkv()
    with pytest.raises(ValueError, match="S holds"):
        ab.ab_select(P, t["Q"], t["K"], _t(B * H * nQ * nK - 1), WS)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ab.ab_select(P, t["Q"], t["K"], _t(B * H * nQ * nK), WS)


def test_select_debug_sizes():
    t = _qkv()
    S = _t(B * H * nQ * nK)
    with pytest.raises(ValueError, match="labels holds"):
        ab.ab_select_debug(P, t["Q"], t["K"], S, WS, labels=_t(B * H * nQ * 128 - 1, torch.int8))
    with pytest.raises(ValueError, match="cent holds"):
        ab.ab_select_debug(P, t["Q"], t["K"], S, WS, cent=_t(B * H * nQ * 8 * d - 1, torch.bfloat16))
    with pytest.raises(ValueError, match="Kp holds"):
        ab.ab_select_debug(P, t["Q"], t["K"], S, WS, Kp=_t(B * H * nK * d - 1, torch.bfloat16))


def test_plan_and_sample_sizes():
    S = _t(B * H * nQ * nK)
    with pytest.raises(ValueError, match="idx holds"):
        ab.ab_plan(P, S, s, 1, 0, _t(B * H * nQ * s - 1, torch.int32), _t(B * H * nQ * s))
    with pytest.raises(ValueError, match="logpi holds"):
        ab.ab_sample(P, S, s, 1, 0, _t(B * H * nQ * s, torch.int32), _t(B * H * nQ * s - 1))
    with pytest.raises(ValueError, match="S holds"):
        ab.ab_plan_variant(P, _t(B * H * nQ * nK - 1), s, 1, 0, "topk",
                           _t(B * H * nQ * s, torch.int32), _t(B * H * nQ * s))
    # the uniform variant reads no scores
    with pytest.raises(ValueError, match="CUDA tensor"):
        ab.ab_plan_variant(P, None, s, 1, 0, "uniform", _t(B * H * nQ * s, torch.int32),
                           _t(B * H * nQ * s))


def test_attention_sizes():
    idx, lp = _t(B * H * nQ * s, torch.int32), _t(B * H * nQ * s)
    for short in ("Q", "K", "V", "O"):
        t = _qkv(short)
        with pytest.raises(ValueError, match=f"{short} holds"):
            ab.ab_attn(P, t["Q"], t["K"], t["V"], idx, lp, s, t["O"])
        with pytest.raises(ValueError, match=f"{short} holds"):
            ab.ab_attn_dense(P, t["Q"], t["K"], t["V"], t["O"])
    t = _qkv()
    with pytest.raises(ValueError, match="idx holds"):
        ab.ab_attn(P, t["Q"], t["K"], t["V"], idx[:-1], lp, s, t["O"])
    with pytest.raises(ValueError, match="trace holds"):
        ab.ab_attn_debug(P, t["Q"], t["K"], t["V"], idx, lp, s, t["O"], 0, 10**9,
                         trace=_t(3 * 16 * 128 - 1, torch.int64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        ab.ab_attn(P, t["Q"], t["K"], t["V"], idx, lp, s, t["O"])


def test_invalid_params_left_to_the_library():
    bad = ab.params(B, H, 0, d, kv_block=bk)
    t = _qkv()
    with pytest.raises(ValueError, match="CUDA tensor"):  # no size error for N = 0
        ab.ab_attn_dense(bad, t["Q"], t["K"], t["V"], t["O"])
