"""The FMA-pipe exp2 used for part of the selector's exponentials (csrc/common.cuh).

The polynomial's coefficients are read from the source and evaluated the way the kernel
evaluates them (fp32 range reduction with the 1.5 * 2^23 rounding constant, Horner in
fp32, 2^j added into the exponent field); the result must stay within 3e-7 relative of
2^x, the accuracy class of the MUFU's ex2.approx, over the whole clamped range.
"""

import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "block_sparse_attention_ibcs_b200", "csrc",
                   "common.cuh")


def _coeffs():
    text = open(SRC).read()
    c = {int(k): float(v) for k, v in re.findall(r"EXP2P_C(\d) = ([0-9.e+-]+)f;", text)}
    assert sorted(c) == list(range(6))
    return [np.float32(c[k]) for k in range(6)]


def _fma32(a, b, c):
    # fp32 fused multiply-add: the fp32 x fp32 product is exact in fp64
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly(x):
    x = np.clip(x.astype(np.float32), np.float32(-126), np.float32(127))
    rnd = np.float32(12582912.0)
    t = (x + rnd).astype(np.float32)
    j = (t - rnd).astype(np.float32)
    f = _fma32(j, np.float32(-1), x)
    c = _coeffs()
    p = _fma32(np.full_like(f, c[5]), f, np.full_like(f, c[4]))
    for k in (3, 2, 1, 0):
        p = _fma32(p, f, np.full_like(f, c[k]))
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_exp2_poly_relative_error():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.9, 126.9, 2_000_001, dtype=np.float32),
                        rng.uniform(-30, 30, 1_000_000).astype(np.float32),
                        np.arange(-125, 127, dtype=np.float32)])  # exact integers
    got = _exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 3e-7, rel.max()


def test_exp2_poly_reduction_is_exact():
    # x - round(x) is computed exactly and lies in [-1/2, 1/2]
    x = np.linspace(-126, 127, 100_001, dtype=np.float32)
    rnd = np.float32(12582912.0)
    j = ((x + rnd).astype(np.float32) - rnd).astype(np.float32)
    f = _fma32(j, np.float32(-1), x)
    assert np.all(np.abs(f) <= 0.5)
    assert np.array_equal(f.astype(np.float64), x.astype(np.float64) - j.astype(np.float64))
