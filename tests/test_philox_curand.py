"""The oracle's Philox4x32-10 against cuRAND's, run as a library on the host (no GPU).

The planner draws its systematic-sampling origin U from Philox4x32-10 (Salmon et al., SC'11;
the page names no generator, and the plan reading fixes this one).  cuRAND's host generator
of type CURAND_RNG_PSEUDO_PHILOX4_32_10 is an independent implementation of the same block
function.  Its output stream, established empirically: output k is word k mod 4 of block
g = k div 4, and block g is Philox4x32-10 of the counter (g div 65536 as a 64-bit number in
words 0-1, g mod 65536 in word 2, 0 in word 3) under the key (seed low word, seed high
word); the generator offset counts outputs.  The cases below reach counter words 0, 1 and 2
with values up to 65535 and both key words.
"""

import ctypes
import os

import numpy as np
import pytest

from oracle import abattn_oracle as O

CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161
THREADS = 65536


def _curand():
    for path in ("/usr/local/cuda/lib64/libcurand.so", "libcurand.so", "libcurand.so.10"):
        try:
            return ctypes.CDLL(path)
        except OSError:
            continue
    pytest.skip("libcurand not found")


def _stream(seed, offset, n):
    L = _curand()
    gen = ctypes.c_void_p()
    assert L.curandCreateGeneratorHost(ctypes.byref(gen), CURAND_RNG_PSEUDO_PHILOX4_32_10) == 0
    try:
        assert L.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert L.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(offset)) == 0
        buf = (ctypes.c_uint * n)()
        assert L.curandGenerate(gen, buf, ctypes.c_size_t(n)) == 0
        return np.frombuffer(buf, dtype=np.uint32).copy()
    finally:
        L.curandDestroyGenerator(gen)


def _oracle_block(g, seed):
    hi = g // THREADS
    ctr = (hi & 0xFFFFFFFF, hi >> 32, g % THREADS, 0)
    return list(O.philox4x32_10(ctr, (seed & 0xFFFFFFFF, seed >> 32)))


@pytest.mark.parametrize("seed", [0x123456789ABCDEF0, 2, 0xFFFFFFFF00000001])
def test_first_round_and_the_next(seed):
    n = 4 * (THREADS + 16)
    out = _stream(seed, 0, n)
    for g in list(range(16)) + list(range(THREADS - 16, THREADS + 16)):
        assert list(out[4 * g: 4 * g + 4]) == _oracle_block(g, seed), f"block {g}"


def test_offset_reaches_counter_word_1():
    seed = 0x0BADC0DE12345678
    g0 = THREADS * ((1 << 32) + 3) + 7  # counter (3, 1, 7, 0)
    out = _stream(seed, 4 * g0, 4 * 8)
    for b in range(8):
        assert list(out[4 * b: 4 * b + 4]) == _oracle_block(g0 + b, seed), f"block {g0 + b}"


def test_plan_uniform_is_word_0_of_the_row_counter():
    """U of plan row r (offset 0) is word 0 of the block at counter (r, 0, 0, 0): cuRAND's
    block g = r * 65536 under the same seed."""
    seed = 0x00000000DEADBEEF
    for r in (0, 1, 5, 591):
        out = _stream(seed, 4 * r * THREADS, 4)
        assert int(out[0]) == O.plan_uniform(r, seed, 0)
