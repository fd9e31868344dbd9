"""Shared helpers for the GPU parity tests (comparison metrics and tensor plumbing)."""

import numpy as np
import torch

# Tolerances for the attention output O (bf16 inputs, fp32 accumulation, bf16 output)
# against the fp64 oracle on the identical plan.
O_MAX_ABS = 1e-2
O_REL_L2 = 5e-3
# Block scores S: elementwise relative tolerance in fp32 (values below 1e-30 must be
# below 1e-30 on both sides).
S_REL = 1e-4
S_TINY = 1e-30


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_o_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    err = np.abs(got - ref).max()
    r = rel_l2(got, ref)
    assert err <= O_MAX_ABS, f"{what}: max-abs {err:.3e} > {O_MAX_ABS}"
    assert r <= O_REL_L2, f"{what}: rel-L2 {r:.3e} > {O_REL_L2}"
    return err, r


def assert_s_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    big = ref >= S_TINY
    rel = np.abs(got[big] - ref[big]) / ref[big]
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= S_REL, f"{what}: worst relative S error {worst:.3e}"
    assert (np.abs(got[~big]) <= S_TINY).all(), f"{what}: S above 1e-30 where the oracle is tiny"
    return worst


def f32_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    ia = np.asarray(a, dtype=np.float32).view(np.int32).astype(np.int64)
    ib = np.asarray(b, dtype=np.float32).view(np.int32).astype(np.int64)
    return np.abs(ia - ib)
