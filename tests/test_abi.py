"""The C ABI loads, exports every symbol include/abattn.h declares, and validates on the host.

No call here reaches the GPU: each either is pure host code (workspace size, status
strings) or is rejected by host-side validation before any CUDA call.
"""

import ctypes
import os
import re

import pytest

import block_sparse_attention_ibcs_b200 as ab

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "abattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ab_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = ab.lib()
    names = _declared()
    assert {"ab_select", "ab_plan", "ab_attn", "ab_sample", "ab_attn_dense", "ab_get_status",
            "ab_workspace_bytes", "ab_select_debug", "ab_status_string"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    for code, name in ab.STATUS_NAMES.items():
        assert ab.ab_status_string(code)
    assert ab.ab_status_string(12345) == "unknown status"
    assert ab.ab_version() >= 100


def test_workspace_bytes():
    p = ab.params(1, 40, 75600, 128)
    n = ab.ab_workspace_bytes(p)
    nK, nQ = 18900, 591
    groups = -(-nQ // 32)  # the score passes keep 8 key-chunk slots of (m, z) per centroid row
    expect = (40 * nK * 128 * 2 + 40 * nQ * 8 * 128 * 2 + 40 * nQ * 8 * 4
              + 40 * groups * 256 * 8 * 8)
    assert expect <= n <= expect + 4 * 256


@pytest.mark.parametrize("bad,code", [
    (dict(d=96), -2), (dict(d=0), -1), (dict(q_block=64), -2), (dict(kv_block=3), -1),
    (dict(kv_block=256), -1), (dict(clusters=0), -1), (dict(clusters=9), -2),
    (dict(kmeans_iters=-1), -1), (dict(kmeans_iters=5), -2), (dict(N=0), -1),
    (dict(B=0), -1), (dict(H=0), -1), (dict(B=-3), -1),
    # size limits: (b, h, query block) CTAs must fit a 1-D grid, nK * 2^32 a uint64
    (dict(B=1, H=4_000_000, N=75600), -2), (dict(N=(1 << 31) - 1, kv_block=1), -2),
    # head slices: [head0, head0 + H) must lie inside the layer's heads_total heads
    (dict(head0=1), -1), (dict(head0=-1, heads_total=8), -1), (dict(heads_total=-2), -1),
    (dict(head0=7, heads_total=8), -1), (dict(head0=0, heads_total=1), -1),
    # the whole layer's plan rows must fit the 32-bit Philox counter word
    (dict(N=75600, heads_total=4_000_000), -2),
])
def test_bad_params_rejected(bad, code):
    kw = dict(B=1, H=2, N=1024, d=64, kv_block=4, clusters=8, kmeans_iters=1, q_block=128,
              head0=0, heads_total=0)
    kw.update(bad)
    p = ab.ABParams(kw["B"], kw["H"], kw["N"], kw["d"], kw["q_block"], kw["kv_block"],
                    kw["clusters"], kw["kmeans_iters"], kw["head0"], kw["heads_total"])
    n = ctypes.c_size_t(0)
    assert ab.lib().ab_workspace_bytes(ctypes.byref(p), ctypes.byref(n)) == code


@pytest.mark.parametrize("head0,heads_total", [(0, 0), (0, 2), (6, 8), (3, 40)])
def test_head_slices_accepted(head0, heads_total):
    p = ab.params(1, 2, 1024, 64, head0=head0, heads_total=heads_total)
    assert ab.ab_workspace_bytes(p) == ab.ab_workspace_bytes(ab.params(1, 2, 1024, 64))


def test_largest_accepted_grid():
    # BH * nQ = 2^31 - 1 exactly is accepted (one CTA per (b, h, query block))
    nQ = 591
    H = ((1 << 31) - 1) // nQ
    p = ab.params(1, H, 75600, 128)
    n = ctypes.c_size_t(0)
    assert ab.lib().ab_workspace_bytes(ctypes.byref(p), ctypes.byref(n)) == 0
    p = ab.params(1, H + 1, 75600, 128)
    assert ab.lib().ab_workspace_bytes(ctypes.byref(p), ctypes.byref(n)) == -2


def test_null_and_misaligned_pointers_rejected_before_any_cuda_call():
    L = ab.lib()
    p = ab.params(1, 2, 1024, 64)
    P = ctypes.byref(p)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    odd = ctypes.c_void_p(0x10008)
    null = ctypes.c_void_p(0)
    assert L.ab_select(P, null, fake, fake, fake, 1 << 30, null) == -1
    assert L.ab_select(P, fake, fake, fake, null, 1 << 30, null) == -5
    assert L.ab_select(P, fake, fake, fake, ctypes.c_void_p(0x10010), 1 << 30, null) == -5
    assert L.ab_select(P, fake, fake, fake, fake, 16, null) == -5  # workspace too small
    assert L.ab_attn(P, fake, fake, odd, fake, fake, 32, fake, null) == -1
    assert L.ab_attn(P, fake, fake, fake, null, fake, 32, fake, null) == -1
    assert L.ab_attn(P, fake, fake, fake, fake, fake, 0, fake, null) == -1  # s < 1
    assert L.ab_attn(P, fake, fake, fake, fake, fake, 257, fake, null) == -1  # s > nK
    assert L.ab_plan(P, null, 32, 1, 0, fake, fake, null) == -1
    assert L.ab_plan(P, fake, 0, 1, 0, fake, fake, null) == -1
    assert L.ab_plan(P, fake, 300, 1, 0, fake, fake, null) == -1
    assert L.ab_sample(P, fake, 32, 1, 0, null, fake, null) == -1
    assert L.ab_select_plan(P, fake, fake, fake, fake, 1 << 30, 0, 1, 0, fake, fake, 0, null,
                            null) == -1                                     # s < 1
    assert L.ab_select_plan(P, fake, fake, fake, null, 1 << 30, 32, 1, 0, fake, fake, 0, null,
                            null) == -5                                     # no workspace
    assert L.ab_select_plan(P, fake, fake, fake, fake, 16, 32, 1, 0, fake, fake, 0, null,
                            null) == -5                                     # workspace too small
    assert L.ab_plan_variant(P, fake, 32, 1, 0, 7, fake, fake, null) == -1   # unknown mode
    assert L.ab_plan_variant(P, fake, 32, 1, 0, -1, fake, fake, null) == -1
    assert L.ab_plan_variant(P, null, 32, 1, 0, 3, fake, fake, null) == -1   # top-k needs S
    assert L.ab_plan_variant(P, fake, 300, 1, 0, 2, fake, fake, null) == -1  # s > nK
    assert L.ab_attn_dense(P, fake, null, fake, fake, null) == -1
    assert L.ab_attn(None, fake, fake, fake, fake, fake, 32, fake, null) == -1
