"""ab_select_noalloc: the selector for callers that cannot allocate device memory.

Such callers (a plugin whose host framework owns all device memory, a serving loop whose
memory plan is frozen at start-up) have no workspace to pass, so the library keeps the
selector's scratch in one built-in array.  This file is collected last on purpose: the
array is shared by every call, and the test must hold both in a fresh process and after
all other tests have run.
"""

import ctypes

import pytest
import torch

import block_sparse_attention_ibcs_b200 as ab
from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, gaussian_head, make_qkv

from _util import assert_s_close


def _with_workspace(p, Q, K, shape):
    S = torch.empty(shape, device="cuda")
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    ab.ab_select(p, Q, K, S, ws)
    return S


@pytest.mark.gpu
def test_noalloc_matches_workspace_select_on_two_calls_in_a_row():
    # call 1: the tiny configuration
    w = WORKLOADS["tiny"]
    Q1, K1, _ = (t.cuda() for t in make_qkv(w))
    p1 = ab.params(w.B, w.H, w.N, w.d, w.kv_block)
    shape1 = (w.B, w.H, w.nQ, w.nK)
    # call 2: another shape (ragged blocks, d = 128), so the shared scratch holds stale data
    N2, d2 = 1000, 128
    Q2 = torch.stack([gaussian_head(N2, d2, 301 + h) for h in range(3)])[None].bfloat16().cuda()
    K2 = torch.stack([gaussian_head(N2, d2, 401 + h) for h in range(3)])[None].bfloat16().cuda()
    p2 = ab.params(1, 3, N2, d2, kv_block=16)
    shape2 = (1, 3, 8, 63)

    S1 = torch.full(shape1, float("nan"), device="cuda")
    S2 = torch.full(shape2, float("nan"), device="cuda")
    ab.ab_select_noalloc(p1, Q1, K1, S1)
    ab.ab_select_noalloc(p2, Q2, K2, S2)
    assert ab.ab_get_status() == 0
    R1 = _with_workspace(p1, Q1, K1, shape1)
    R2 = _with_workspace(p2, Q2, K2, shape2)
    assert ab.ab_get_status() == 0
    # the same kernels with the same work split: S must match bit for bit (stale scratch
    # left by call 1 must not leak into call 2)
    assert torch.equal(S1, R1), "no-alloc call 1 differs from ab_select"
    assert torch.equal(S2, R2), "no-alloc call 2 differs from ab_select"
    assert_s_close(S1.cpu().numpy(), R1.cpu().double().numpy(), "no-alloc call 1")
    assert_s_close(S2.cpu().numpy(), R2.cpu().double().numpy(), "no-alloc call 2")


def test_noalloc_rejects_shapes_beyond_the_builtin_scratch():
    # host-side check only: returns before touching any device
    p = ab.params(1, 40, 75600, 128)
    f = ab.lib().ab_select_noalloc
    f.argtypes = [ctypes.POINTER(ab.ABParams)] + [ctypes.c_void_p] * 4
    f.restype = ctypes.c_int
    fake = ctypes.c_void_p(0x10000)
    assert f(ctypes.byref(p), fake, fake, fake, None) == -5
