"""B200-native AB-Attention hot path: thin Python binding over ``libabattn.so``.

Every function here only marshals arguments (torch tensors -> device pointers, the
current CUDA stream) and calls the C ABI declared in ``include/abattn.h``; all
computation runs in the library's sm_100a kernels.  There is no CPU fallback: if
the library is missing, calls raise.

The three stages of AB-Attention (onedev.kr/papers/1521):
  ab_select(Q, K) -> S           IBCS block scores
  ab_plan(S, s, seed) -> idx, logpi   SIP inclusion probabilities + systematic sampling
  ab_attn(Q, K, V, idx, logpi) -> O   packed-tile attention with the -log(pi) shift
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "ABError", "ABParams", "params", "lib", "ab_workspace_bytes", "ab_select",
    "ab_select_debug", "ab_select_plan", "ab_plan", "ab_plan_variant", "ab_sample", "ab_attn",
    "ab_attn_dense", "ab_attn_debug", "ab_select_noalloc",
    "ab_get_status", "ab_status_string", "ab_version", "LIB_PATH", "PLAN_MODES",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libabattn.so")

AB_OK = 0
# ab_plan_mode (include/abattn.h): planner variants for the page's ablations
PLAN_MODES = {"sip": 0, "sip_no_ipw": 1, "uniform": 2, "topk": 3}
STATUS_NAMES = {
    0: "AB_OK", -1: "AB_ERR_INVALID_ARG", -2: "AB_ERR_UNSUPPORTED", -3: "AB_ERR_CUDA",
    -4: "AB_ERR_DEVICE_TIMEOUT", -5: "AB_ERR_WORKSPACE", -6: "AB_ERR_NOT_IMPLEMENTED",
    -7: "AB_ERR_DEVICE_CHECK",
}


class ABError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({ab_status_string(code)})")


class ABParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("B", "H", "N", "d", "q_block", "kv_block", "clusters", "kmeans_iters", "head0",
                 "heads_total")]


def params(B, H, N, d, kv_block=4, clusters=8, kmeans_iters=1, q_block=128, head0=0,
           heads_total=0) -> ABParams:
    """Parameters of a call over heads [head0, head0 + H) of a layer of heads_total heads
    (heads_total = 0: the call is the whole layer)."""
    return ABParams(B, H, N, d, q_block, kv_block, clusters, kmeans_iters, head0, heads_total)


_LIB = None
_P = ctypes.POINTER(ABParams)
_vp, _sz, _i, _u64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint64

_SIGS = {
    "ab_workspace_bytes": [_P, ctypes.POINTER(_sz)],
    "ab_select": [_P, _vp, _vp, _vp, _vp, _sz, _vp],
    "ab_select_debug": [_P, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp, _vp, _vp],
    "ab_plan": [_P, _vp, _i, _u64, _u64, _vp, _vp, _vp],
    "ab_plan_variant": [_P, _vp, _i, _u64, _u64, _i, _vp, _vp, _vp],
    "ab_select_plan": [_P, _vp, _vp, _vp, _vp, _sz, _i, _u64, _u64, _vp, _vp, _i, _vp, _vp],
    "ab_sample": [_P, _vp, _i, _u64, _u64, _vp, _vp, _vp],
    "ab_attn": [_P, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp],
    "ab_attn_dense": [_P, _vp, _vp, _vp, _vp, _vp],
    "ab_attn_debug": [_P, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _u64, _vp, _vp],
    "ab_get_status": [_vp],
    "ab_status_string": [_i],
    "ab_version": [],
}


def lib() -> ctypes.CDLL:
    """Load the in-tree library (built by ``__graft_entry__.build()``)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libabattn.so not built ({LIB_PATH}); run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, argt in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = argt
            f.restype = ctypes.c_char_p if name == "ab_status_string" else ctypes.c_int
        _LIB = L
    return _LIB


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t, name, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _sizes(p):
    """(B*H, nQ, nK) of a parameter set, or None when the parameters are invalid (the
    library then reports that itself)."""
    if p is None or min(p.B, p.H, p.N, p.d, p.kv_block) < 1:
        return None
    return p.B * p.H, -(-p.N // 128), -(-p.N // p.kv_block)


def _need(p, **bufs):
    """Every given tensor holds at least the elements the call reads or writes through its
    pointer; ``bufs`` maps a name to (tensor, count as a function of (BH, nQ, nK)).  A smaller
    buffer would send the kernels past its end, so it is refused here."""
    dims = _sizes(p)
    if dims is None:
        return
    for name, (t, count) in bufs.items():
        if t is None:
            continue
        n = int(count(*dims))
        if t.numel() < n:
            raise ValueError(f"{name} holds {t.numel()} elements; the call needs {n}")


def _qkv(p, *names_tensors):
    """Size rules for [B,H,N,d] tensors."""
    return {n: (t, lambda bh, nq, nk: bh * p.N * p.d) for n, t in names_tensors}


def _check(code: int, where: str):
    if code != AB_OK:
        raise ABError(code, where)


def ab_status_string(code: int) -> str:
    return lib().ab_status_string(int(code)).decode()


def ab_version() -> int:
    return lib().ab_version()


def ab_workspace_bytes(p: ABParams) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ab_workspace_bytes(ctypes.byref(p), ctypes.byref(n)), "ab_workspace_bytes")
    return n.value


def ab_select(p, Q, K, S, ws, stream=None):
    import torch

    _need(p, **_qkv(p, ("Q", Q), ("K", K)), S=(S, lambda bh, nq, nk: bh * nq * nk))

    _check(lib().ab_select(ctypes.byref(p), _ptr(Q, "Q", torch.bfloat16), _ptr(K, "K", torch.bfloat16),
                           _ptr(S, "S", torch.float32), _ptr(ws, "ws"), ws.numel() * ws.element_size(),
                           _stream(stream)), "ab_select")


def ab_select_debug(p, Q, K, S, ws, labels=None, cent=None, w=None, Kp=None, stream=None):
    import torch

    _need(p, **_qkv(p, ("Q", Q), ("K", K)), S=(S, lambda bh, nq, nk: bh * nq * nk),
          labels=(labels, lambda bh, nq, nk: bh * nq * 128),
          cent=(cent, lambda bh, nq, nk: bh * nq * p.clusters * p.d),
          w=(w, lambda bh, nq, nk: bh * nq * p.clusters),
          Kp=(Kp, lambda bh, nq, nk: bh * nk * p.d))

    _check(lib().ab_select_debug(
        ctypes.byref(p), _ptr(Q, "Q", torch.bfloat16), _ptr(K, "K", torch.bfloat16),
        _ptr(S, "S", torch.float32), _ptr(ws, "ws"), ws.numel() * ws.element_size(),
        _ptr(labels, "labels", torch.int8), _ptr(cent, "cent", torch.bfloat16),
        _ptr(w, "w", torch.float32), _ptr(Kp, "Kp", torch.bfloat16), _stream(stream)),
        "ab_select_debug")


def ab_plan(p, S, s, seed, offset, idx, logpi, stream=None):
    import torch

    _need(p, S=(S, lambda bh, nq, nk: bh * nq * nk), idx=(idx, lambda bh, nq, nk: bh * nq * s),
          logpi=(logpi, lambda bh, nq, nk: bh * nq * s))

    _check(lib().ab_plan(ctypes.byref(p), _ptr(S, "S", torch.float32), int(s), int(seed), int(offset),
                         _ptr(idx, "idx", torch.int32), _ptr(logpi, "logpi", torch.float32),
                         _stream(stream)), "ab_plan")


def ab_select_plan(p, Q, K, S, ws, s, seed, offset, idx, logpi, groups=0, stream=None,
                   stream2=None):
    """ab_select then ab_plan, overlapped across head groups on ``stream`` and ``stream2``."""
    import torch

    _need(p, **_qkv(p, ("Q", Q), ("K", K)), S=(S, lambda bh, nq, nk: bh * nq * nk),
          idx=(idx, lambda bh, nq, nk: bh * nq * s), logpi=(logpi, lambda bh, nq, nk: bh * nq * s))

    _check(lib().ab_select_plan(ctypes.byref(p), _ptr(Q, "Q", torch.bfloat16),
                                _ptr(K, "K", torch.bfloat16), _ptr(S, "S", torch.float32),
                                _ptr(ws, "ws"), ws.numel() * ws.element_size(), int(s), int(seed),
                                int(offset), _ptr(idx, "idx", torch.int32),
                                _ptr(logpi, "logpi", torch.float32), int(groups), _stream(stream),
                                None if stream2 is None else _stream(stream2)), "ab_select_plan")


def ab_plan_variant(p, S, s, seed, offset, mode, idx, logpi, stream=None):
    """Planner variant ``mode`` (a name in PLAN_MODES or its number); S may be None for
    "uniform"."""
    import torch

    _need(p, S=(S, lambda bh, nq, nk: bh * nq * nk), idx=(idx, lambda bh, nq, nk: bh * nq * s),
          logpi=(logpi, lambda bh, nq, nk: bh * nq * s))

    m = PLAN_MODES[mode] if isinstance(mode, str) else int(mode)
    _check(lib().ab_plan_variant(ctypes.byref(p), _ptr(S, "S", torch.float32), int(s), int(seed),
                                 int(offset), m, _ptr(idx, "idx", torch.int32),
                                 _ptr(logpi, "logpi", torch.float32), _stream(stream)),
           "ab_plan_variant")


def ab_sample(p, pi, s, seed, offset, idx, logpi, stream=None):
    import torch

    _need(p, pi=(pi, lambda bh, nq, nk: bh * nq * nk), idx=(idx, lambda bh, nq, nk: bh * nq * s),
          logpi=(logpi, lambda bh, nq, nk: bh * nq * s))

    _check(lib().ab_sample(ctypes.byref(p), _ptr(pi, "pi", torch.float32), int(s), int(seed),
                           int(offset), _ptr(idx, "idx", torch.int32),
                           _ptr(logpi, "logpi", torch.float32), _stream(stream)), "ab_sample")


def ab_attn(p, Q, K, V, idx, logpi, s, O, stream=None):
    import torch

    _need(p, **_qkv(p, ("Q", Q), ("K", K), ("V", V), ("O", O)),
          idx=(idx, lambda bh, nq, nk: bh * nq * s), logpi=(logpi, lambda bh, nq, nk: bh * nq * s))

    bf = torch.bfloat16
    _check(lib().ab_attn(ctypes.byref(p), _ptr(Q, "Q", bf), _ptr(K, "K", bf), _ptr(V, "V", bf),
                         _ptr(idx, "idx", torch.int32), _ptr(logpi, "logpi", torch.float32), int(s),
                         _ptr(O, "O", bf), _stream(stream)), "ab_attn")


def ab_attn_dense(p, Q, K, V, O, stream=None):
    import torch

    _need(p, **_qkv(p, ("Q", Q), ("K", K), ("V", V), ("O", O)))

    bf = torch.bfloat16
    _check(lib().ab_attn_dense(ctypes.byref(p), _ptr(Q, "Q", bf), _ptr(K, "K", bf), _ptr(V, "V", bf),
                               _ptr(O, "O", bf), _stream(stream)), "ab_attn_dense")


def ab_attn_debug(p, Q, K, V, idx, logpi, s, O, skip_first_arrival, timeout_ns, trace=None,
                  stream=None):
    """Test/profiling hook: ab_attn with a producer arrival skipped, another device wait
    limit, and optionally a per-tile clock64 event trace (int64 tensor of 3*16*128)."""
    import torch

    _need(p, **_qkv(p, ("Q", Q), ("K", K), ("V", V), ("O", O)),
          idx=(idx, lambda bh, nq, nk: bh * nq * s), logpi=(logpi, lambda bh, nq, nk: bh * nq * s),
          trace=(trace, lambda bh, nq, nk: 3 * 16 * 128))

    bf = torch.bfloat16
    _check(lib().ab_attn_debug(ctypes.byref(p), _ptr(Q, "Q", bf), _ptr(K, "K", bf), _ptr(V, "V", bf),
                               _ptr(idx, "idx", torch.int32), _ptr(logpi, "logpi", torch.float32),
                               int(s), _ptr(O, "O", bf), int(skip_first_arrival), int(timeout_ns),
                               _ptr(trace, "trace", torch.int64), _stream(stream)), "ab_attn_debug")


def ab_get_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return lib().ab_get_status(_stream(stream))


def ab_select_noalloc(p, Q, K, S, stream=None):
    """ab_select without a workspace: the library's built-in scratch (16 MiB per GPU) is used.

    For callers that may not allocate device memory and have no scratch buffer to pass.
    Calls that overlap on the GPU share that scratch and race; serialise them.
    """
    import torch

    _need(p, **_qkv(p, ("Q", Q), ("K", K)), S=(S, lambda bh, nq, nk: bh * nq * nk))

    f = lib().ab_select_noalloc
    f.argtypes = [_P, _vp, _vp, _vp, _vp]
    f.restype = ctypes.c_int
    _check(f(ctypes.byref(p), _ptr(Q, "Q", torch.bfloat16), _ptr(K, "K", torch.bfloat16),
             _ptr(S, "S", torch.float32), _stream(stream)), "ab_select_noalloc")
