"""Pins for the CPU oracle: it is checked against things other than itself.

Each test fixes one part of the oracle by what the AB-Attention page
(onedev.kr/papers/1521) or plain mathematics determines: closed forms, exact
enumeration, library routines for special cases, hand-worked examples and
invariants.  None of these calls the CUDA library.
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import abattn_oracle as O

TWO32 = 1 << 32


# ---------------------------------------------------------------- bf16 rounding


def _nearest_bf16_exact(x: float) -> float:
    """Brute force: the two bf16 neighbours of x by exact rationals, ties to even."""
    if x == 0:
        return 0.0
    sgn = -1.0 if x < 0 else 1.0
    ax = Fraction(abs(x))
    e = math.floor(math.log2(abs(x)))
    while Fraction(2) ** e > ax:
        e -= 1
    while Fraction(2) ** (e + 1) <= ax:
        e += 1
    ulp = Fraction(2) ** (e - 7)
    k = ax // ulp
    lo, hi = k * ulp, (k + 1) * ulp
    if ax - lo < hi - ax:
        r = lo
    elif ax - lo > hi - ax:
        r = hi
    else:
        r = lo if k % 2 == 0 else hi
    return sgn * float(r)


def test_bf16_round_matches_exact_nearest():
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-20, 20, 2000),
                         rng.standard_normal(200)])
    got = O.bf16_round(xs)
    for x, g in zip(xs, got):
        assert g == _nearest_bf16_exact(float(x)), x


def test_bf16_round_ties_to_even():
    # midpoints between adjacent bf16 values are exact in fp64
    for k in range(128, 256):
        lo = k / 128.0
        mid = (k + 0.5) / 128.0
        want = lo if k % 2 == 0 else (k + 1) / 128.0
        assert O.bf16_round(np.array([mid]))[0] == want
        assert O.bf16_round(np.array([-mid]))[0] == -want


def test_bf16_round_agrees_with_torch_on_fp32_inputs():
    # torch's fp32 -> bf16 cast is round-to-nearest-even; on fp32-representable values
    # a single rounding from fp64 must agree with it.
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(100000, generator=g) * 3).float()
    want = x.bfloat16().double().numpy()
    got = O.bf16_round(x.double().numpy())
    assert np.array_equal(got, want)


def test_bf16_round_specials():
    assert O.bf16_round(np.array([3.5e38]))[0] == np.inf  # beyond the largest finite bf16
    sub = 2.0 ** -133
    assert O.bf16_round(np.array([1.5 * sub]))[0] == 2 * sub  # subnormal tie to even
    assert O.bf16_round(np.array([2.5 * sub]))[0] == 2 * sub
    assert np.isnan(O.bf16_round(np.array([np.nan]))[0])


# ---------------------------------------------------------------- pooling / k-means


def test_pool_keys_hand_example():
    # N = 10 keys, d = 2, blocks of 4: last block holds 2 valid keys (mean over 2).
    K = np.stack([np.arange(10.0), 2 * np.arange(10.0)], 1)
    Kp = O.pool_keys(K, 4)
    assert Kp.shape == (3, 2)
    assert np.array_equal(Kp, [[1.5, 3.0], [5.5, 11.0], [8.5, 17.0]])


def test_kmeans_hand_example():
    # n = 4 one-dimensional queries, 2 clusters.  Segment means: {0,1} -> 0.5, {2,10} -> 6.
    # Query 2 is nearer 0.5 (1.5 < 4), so it moves: clusters {0,1,2}, {10}.
    Qb = np.array([[0.0], [1.0], [2.0], [10.0]])
    cent, w, labels, _ = O.kmeans_block(Qb, C=2, iters=1)
    assert labels.tolist() == [0, 0, 0, 1]
    assert cent[:, 0].tolist() == [1.0, 10.0]
    assert w.tolist() == [0.75, 0.25]
    # zero iterations: the position-based segment means of the ablation paragraph
    cent0, w0, labels0, _ = O.kmeans_block(Qb, C=2, iters=0)
    assert cent0[:, 0].tolist() == [0.5, 6.0] and w0.tolist() == [0.5, 0.5]
    assert labels0.tolist() == [0, 0, 1, 1]


def test_kmeans_invariants_random_blocks():
    rng = np.random.default_rng(2)
    for n in (128, 80, 16, 5):
        Qb = O.bf16_round(rng.standard_normal((n, 64)) + rng.integers(0, 3, (n, 1)))
        cent, w, labels, gap = O.kmeans_block(Qb, 8, 1)
        assert abs(w.sum() - 1.0) < 1e-15
        # initial centroids by brute force, then nearest-centroid property of the labels
        init = []
        for c in range(8):
            a, b = c * n // 8, (c + 1) * n // 8
            init.append(Qb[a:b].mean(0) if b > a else None)
        for r in range(n):
            dists = [np.inf if ci is None else float(((Qb[r] - ci) ** 2).sum()) for ci in init]
            best = min(dists)
            assert dists[labels[r]] <= best * (1 + 1e-12)
        for c in range(8):
            mem = Qb[labels == c]
            if len(mem):
                assert np.array_equal(cent[c], O.bf16_round(mem.mean(0)))
                assert w[c] == len(mem) / n
            else:
                assert w[c] == 0 and not cent[c].any()


def test_kmeans_identical_queries():
    q = O.bf16_round(np.random.default_rng(3).standard_normal(32))
    Qb = np.tile(q, (128, 1))
    cent, w, labels, _ = O.kmeans_block(Qb, 8, 1)
    assert w[0] == 1.0 and (labels == 0).all() and np.array_equal(cent[0], q)


def test_kmeans_gap_hand_example():
    # n = 6 one-dimensional queries, 3 clusters: segments {0,2}, {-1,-3}, {9,11} have means
    # 1, -2, 10.  Query 0 lies at squared distances 1, 4, 100: the best and the second best
    # give (4 - 1) / 4 = 0.75 (the third distance must not enter).
    Qb = np.array([[0.0], [2.0], [-1.0], [-3.0], [9.0], [11.0]])
    _, _, labels, gap = O.kmeans_block(Qb, C=3, iters=1)
    assert labels.tolist() == [0, 0, 1, 1, 2, 2]
    # distances: q1 = 2: 1, 16, 64; q2 = -1: 4, 1, 121; q3 = -3: 16, 1, 169; q4 = 9: 64, 121,
    # 1; q5 = 11: 100, 169, 1
    assert gap.tolist() == [0.75, 15 / 16, 0.75, 15 / 16, 63 / 64, 99 / 100]


def test_kmeans_gap_exact_tie_is_zero():
    # segments {-3, 3}, {3, 9} have means 0 and 6; both queries at 3 are 9 from each mean:
    # an exact tie (gap 0), resolved to the lower cluster.
    Qb = np.array([[-3.0], [3.0], [3.0], [9.0]])
    cent, w, labels, gap = O.kmeans_block(Qb, C=2, iters=1)
    assert labels.tolist() == [0, 0, 0, 1]
    assert gap.tolist() == [72 / 81, 0.0, 0.0, 72 / 81]
    assert w.tolist() == [0.75, 0.25] and cent[:, 0].tolist() == [1.0, 9.0]


def test_kmeans_gap_ignores_emptied_clusters():
    # segments {0}, {10}, {9, 11}: means 0, 10, 10.  The first assignment sends 10, 9 and 11
    # to cluster 1 (ties to the lower index), so cluster 2 empties.  In the second
    # assignment query 9 is 81 from cluster 0 and 1 from cluster 1; the emptied cluster
    # (its old mean 10 would also be at distance 1) must not count: gap = 80/81, not 0.
    Qb = np.array([[0.0], [10.0], [9.0], [11.0]])
    cent, w, labels, gap = O.kmeans_block(Qb, C=3, iters=2)
    assert labels.tolist() == [0, 1, 1, 1]
    assert w.tolist() == [0.25, 0.75, 0.0]
    assert cent[:, 0].tolist() == [0.0, 10.0, 0.0]
    assert gap.tolist() == [1.0, 1.0, 80 / 81, 120 / 121]
    # only one live cluster: no runner-up, so no near-tie
    _, _, _, g1 = O.kmeans_block(np.array([[1.0], [1.0]]), C=2, iters=2)
    assert np.isinf(g1).all()


def test_scores_from_labels_hand_example():
    # d = 1, two pooled keys 0 and 1.  Labels put query 1 (value 0) into cluster 1 with the
    # two queries at 2: cluster 0 = {0} (mean 0, share 1/4), cluster 1 = {0, 2, 2} (mean 4/3,
    # share 3/4).  4/3 = 1.0101010...b rounds to the bf16 value 1.0101011b = 1.3359375.
    # With two keys each softmax is a logistic: cluster 0 gives (1/2, 1/2), cluster 1 gives
    # (1 - p, p) with p = 1 / (1 + e^-1.3359375).
    Qb = np.array([[0.0], [0.0], [2.0], [2.0]])
    Kp = np.array([[0.0], [1.0]])
    S = O.scores_from_labels(Qb, np.array([0, 1, 1, 1]), Kp, C=2)
    p = 1.0 / (1.0 + math.exp(-1.3359375))
    want = [0.25 * 0.5 + 0.75 * (1 - p), 0.25 * 0.5 + 0.75 * p]
    assert S.dtype == np.float32
    np.testing.assert_allclose(S, want, rtol=2e-7, atol=0)
    # the unrounded mean 4/3 would be off by far more than the fp32 output rounding
    p_raw = 1.0 / (1.0 + math.exp(-4.0 / 3.0))
    assert abs(0.75 * (p - p_raw)) > 1e-4 * want[1]


def test_scores_from_labels_reproduces_kmeans_scores():
    # with the labels of the last assignment, the rebuilt centroids and shares are exactly
    # kmeans_block's, so the score rows agree bit for bit (iterations 0, 1, 2; ragged n)
    rng = np.random.default_rng(6)
    Kp = O.bf16_round(rng.standard_normal((200, 32)))
    for n in (128, 80, 13):
        Qb = O.bf16_round(rng.standard_normal((n, 32)) + rng.integers(0, 4, (n, 1)))
        for iters in (0, 1, 2):
            cent, w, labels, _ = O.kmeans_block(Qb, 8, iters)
            want = O.block_scores(cent, w, Kp).astype(np.float32)
            got = O.scores_from_labels(Qb, labels, Kp, C=8)
            assert np.array_equal(got, want), (n, iters)


# ---------------------------------------------------------------- scores


def test_scores_sum_to_one_and_single_cluster_is_softmax():
    from scipy.special import softmax

    rng = np.random.default_rng(4)
    Kp = O.bf16_round(rng.standard_normal((300, 64)))
    cent = O.bf16_round(rng.standard_normal((8, 64)))
    w = rng.dirichlet(np.ones(8))
    S = O.block_scores(cent, w, Kp)
    assert abs(S.sum() - 1) < 1e-12
    one = O.block_scores(cent[:1], np.array([1.0]), Kp)
    assert np.allclose(one, softmax(cent[0] @ Kp.T / 8.0), rtol=1e-13, atol=0)


def test_select_identical_queries_gives_softmax_of_mean():
    from scipy.special import softmax

    rng = np.random.default_rng(5)
    q = O.bf16_round(rng.standard_normal(64))
    Qh = np.tile(q, (256, 1))
    Kh = O.bf16_round(rng.standard_normal((256, 64)))
    S = O.select_head(Qh, Kh, 128, 4, 8, 1)
    Kp = np.array([O.bf16_round(Kh[4 * j:4 * j + 4].mean(0)) for j in range(64)])
    want = softmax(q @ Kp.T / 8.0)
    assert np.allclose(S[0], want, rtol=1e-6, atol=0) and np.allclose(S[1], want, rtol=1e-6)


# ---------------------------------------------------------------- λ and π


def _water_fill_exact(S, s):
    """Closed-form λ of Σ_j min(1, λ S_j) = s by sorting (exact rationals)."""
    v = sorted((Fraction(float(x)) for x in S if x > 0), reverse=True)
    tail = sum(v, Fraction(0))
    for k in range(len(v) + 1):  # k blocks saturated
        if k > s:
            break
        lam = Fraction(s - k) / tail if tail > 0 else None
        if lam is not None and (k == 0 or lam * v[k - 1] >= 1) and (k == len(v) or lam * v[k] < 1):
            return lam
        if k < len(v):
            tail -= v[k]
    return None


@pytest.mark.parametrize("seed,nK,s,sigma", [(0, 256, 32, 2.0), (1, 2000, 200, 3.0),
                                             (2, 500, 10, 0.3), (3, 300, 299, 1.0)])
def test_lambda_matches_water_filling(seed, nK, s, sigma):
    rng = np.random.default_rng(seed)
    x = np.exp(sigma * rng.standard_normal(nK))
    S = (x / x.sum()).astype(np.float32)
    lam_bits = O.solve_lambda(S, s)
    lam = float(O.f32_from_bits(lam_bits))
    exact = _water_fill_exact(S, s)
    assert abs(lam - float(exact)) <= 4e-7 * float(exact)
    g = sum(min(1.0, lam * float(v)) for v in S)
    assert abs(g - s) <= 1e-5 * s


def test_lambda_without_saturation_is_s():
    S = np.full(1000, 1e-3, dtype=np.float32)  # Σ S ≈ 1, s max S ≤ 1
    lam = float(O.f32_from_bits(O.solve_lambda(S, 100)))
    assert abs(lam * float(S.astype(np.float64).sum()) - 100) <= 100 * 4e-7


def test_fixed_point_budget_exact_and_saturation():
    rng = np.random.default_rng(6)
    for trial in range(20):
        nK = int(rng.integers(50, 3000))
        s = int(rng.integers(1, nK))
        x = np.exp(2.5 * rng.standard_normal(nK))
        S = (x / x.sum()).astype(np.float32)
        qp, order, lam_bits = O.inclusion_fixed_point(S, s)
        assert int(qp.sum()) == s * TWO32
        assert (qp <= TWO32).all()
        lam = O.f32_from_bits(lam_bits)
        sat = (np.float32(lam) * S).astype(np.float32) >= 1
        assert (qp[sat] == TWO32).all()  # π = 1 blocks are untouched by the cap


def test_fewer_positive_blocks_than_budget():
    S = np.zeros(50, dtype=np.float32)
    S[[3, 7, 40]] = [0.5, 0.25, 0.25]
    idx, logpi, qp = O.plan_row(S, 6, 1, 0, 0)
    assert idx.tolist() == [0, 1, 2, 3, 7, 40]  # every positive block + the lowest zero blocks
    assert (logpi == 0).all() and int(qp.sum()) == 6 * TWO32


# ---------------------------------------------------------------- systematic sampling


def _pieces(qp, order):
    """U-breakpoints of the systematic sample: the sample is constant between them."""
    pts = {0}
    pos = 0
    for j in order:
        pos += int(qp[j])
        pts.add(pos % TWO32)
    return sorted(pts) + [TWO32]


def test_exact_inclusion_probabilities_by_enumeration():
    rng = np.random.default_rng(7)
    nK, s = 64, 9
    x = np.exp(1.5 * rng.standard_normal(nK))
    S = (x / x.sum()).astype(np.float32)
    qp, order, _ = O.inclusion_fixed_point(S, s)
    pts = _pieces(qp, order)
    freq = np.zeros(nK, dtype=object)
    for a, b in zip(pts[:-1], pts[1:]):
        if b <= a:
            continue
        idx = O.systematic_sample(qp, order, a, s)
        assert np.array_equal(idx, O.systematic_sample(qp, order, b - 1, s))  # constant piece
        assert len(idx) == s and len(set(idx.tolist())) == s
        for j in idx:
            freq[j] += b - a
    assert all(int(freq[j]) == int(qp[j]) for j in range(nK))  # P(j in sample) = π'_j exactly


def test_sample_properties_and_monte_carlo():
    rng = np.random.default_rng(8)
    nK, s = 200, 20
    x = np.exp(2.0 * rng.standard_normal(nK))
    S = (x / x.sum()).astype(np.float32)
    hits = np.zeros(nK)
    R = 3000
    for seed in range(R):
        idx, logpi, qp = O.plan_row(S, s, seed, 0, 0)
        assert len(idx) == s and (np.diff(idx) > 0).all()
        assert set(np.flatnonzero(qp == TWO32)) <= set(idx.tolist())
        assert np.allclose(np.exp(logpi.astype(np.float64)), qp[idx].astype(np.float64) / TWO32,
                           rtol=1e-6)
        hits[idx] += 1
    pi = qp.astype(np.float64) / TWO32
    z = (hits / R - pi) / np.sqrt(np.maximum(pi * (1 - pi), 1e-12) / R)
    assert np.abs(z[(pi > 0) & (pi < 1)]).max() < 5.0


def test_horvitz_thompson_unbiased_exact():
    """Exact E over U of the 1/π-weighted numerator and denominator = dense values."""
    rng = np.random.default_rng(9)
    N, d, bk, s = 96, 16, 4, 6
    Qb = O.bf16_round(rng.standard_normal((5, d)))
    K = O.bf16_round(rng.standard_normal((N, d)))
    V = O.bf16_round(rng.standard_normal((N, d)))
    x = np.exp(rng.standard_normal(N // bk))
    S = (x / x.sum()).astype(np.float32)
    qp, order, _ = O.inclusion_fixed_point(S, s)
    assert (qp > 0).all()
    pts = _pieces(qp, order)
    num = np.zeros((5, d))
    den = np.zeros(5)
    for a, b in zip(pts[:-1], pts[1:]):
        if b > a:
            idx = O.systematic_sample(qp, order, a, s)
            n_, d_ = O.ht_estimates(Qb, K, V, idx, qp, bk)
            num += n_ * ((b - a) / TWO32)
            den += d_ * ((b - a) / TWO32)
    z = Qb @ K.T / math.sqrt(d)
    e = np.exp(z - z.max(1, keepdims=True))
    assert np.allclose(num, e @ V, rtol=1e-10, atol=1e-12)
    assert np.allclose(den, e.sum(1), rtol=1e-10)


def test_horvitz_thompson_monte_carlo_over_seeds():
    rng = np.random.default_rng(10)
    N, d, bk, s = 128, 16, 4, 8
    Qb = O.bf16_round(rng.standard_normal((3, d)))
    K = O.bf16_round(rng.standard_normal((N, d)))
    V = O.bf16_round(rng.standard_normal((N, d)))
    x = np.exp(rng.standard_normal(N // bk))
    S = (x / x.sum()).astype(np.float32)
    R = 4000
    num = np.zeros((3, d))
    den = np.zeros(3)
    dens = []
    for seed in range(R):
        idx, _, qp = O.plan_row(S, s, seed, 0, 0)
        n_, d_ = O.ht_estimates(Qb, K, V, idx, qp, bk)
        num += n_ / R
        den += d_ / R
        dens.append(d_)
    z = Qb @ K.T / math.sqrt(d)
    e = np.exp(z - z.max(1, keepdims=True))
    se = np.std(np.array(dens), 0) / math.sqrt(R)
    assert (np.abs(den - e.sum(1)) < 5 * se).all()
    assert np.abs(num - e @ V).max() < 0.1 * np.abs(e @ V).max()


def test_inverse_pi_weighting_is_logit_shift():
    rng = np.random.default_rng(11)
    N, d, bk, s = 256, 32, 4, 12
    Qb = O.bf16_round(rng.standard_normal((7, d)))
    K = O.bf16_round(rng.standard_normal((N, d)))
    V = O.bf16_round(rng.standard_normal((N, d)))
    x = np.exp(2 * rng.standard_normal(N // bk))
    S = (x / x.sum()).astype(np.float32)
    idx, _, qp = O.plan_row(S, s, 5, 0, 0)
    num, den = O.ht_estimates(Qb, K, V, idx, qp, bk)
    lp = np.log(qp[idx].astype(np.float64) / TWO32)  # fp64 logπ, no fp32 storage
    o = O.attn_block(Qb, K, V, idx, lp, bk)
    assert np.allclose(num / den[:, None], o, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- attention


def test_all_blocks_is_dense_attention_and_sdpa():
    rng = np.random.default_rng(12)
    N, d, bk = 250, 64, 4  # ragged last KV block (2 valid tokens)
    nK = -(-N // bk)
    Qh = O.bf16_round(rng.standard_normal((N, d)))
    K = O.bf16_round(rng.standard_normal((N, d)))
    V = O.bf16_round(rng.standard_normal((N, d)))
    S = np.full(nK, 1.0 / nK, dtype=np.float32)
    idx, logpi, qp = O.plan_row(S, nK, 1, 0, 0)
    assert idx.tolist() == list(range(nK)) and (logpi == 0).all()
    o = O.attn_block(Qh[:128], K, V, idx, logpi, bk)
    dense = O.dense_attention(Qh[:128], K, V)
    assert np.allclose(o, dense, rtol=1e-13, atol=1e-14)
    sd = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Qh[:128])[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])
    assert np.allclose(dense, sd[0].numpy(), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- Philox


def test_philox_round_structure_against_numpy_philox4x64():
    """numpy's Philox bit generator is Philox4x64-10; the oracle's generic Philox block
    function, instantiated with the 4x64 constants published by Salmon et al., must
    reproduce it.  (numpy increments the 256-bit counter before each block.)"""
    c64 = dict(w=64, M0=0xD2E7470EE14C6C93, M1=0xCA5A826395121157,
               W0=0x9E3779B97F4A7C15, W1=0xBB67AE8584CAA73B)
    rng = np.random.default_rng(13)
    for _ in range(20):
        key = [int(v) for v in rng.integers(0, 2 ** 63, 2, dtype=np.uint64)]
        ctr = [int(v) for v in rng.integers(0, 2 ** 63, 4, dtype=np.uint64)]
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64),
                              counter=np.array(ctr, dtype=np.uint64))
        got = [int(v) for v in bg.random_raw(4)]
        c1 = list(ctr)
        c1[0] += 1  # no carry for these draws (< 2^63)
        assert got == list(O.philox4(c1, key, 10, **c64))


# ---------------------------------------------------------------- planner variants (R9)

def test_topk_hand_example():
    # scores 0.1 0.3 0.3 -0 +0 NaN 0.2, s = 4: the two 0.3 (j = 1, 2), 0.2 (j = 6), 0.1 (j = 0)
    S = np.array([0.1, 0.3, 0.3, -0.0, 0.0, np.nan, 0.2], np.float32)
    idx, lp = O.topk_row(S, 4)
    assert idx.tolist() == [0, 1, 2, 6] and (lp == 0).all()
    # s = 5 reaches the zeros: +0 ranks above -0
    assert O.topk_row(S, 5)[0].tolist() == [0, 1, 2, 4, 6]
    # s = 7: everything, NaN last
    assert O.topk_row(S, 7)[0].tolist() == list(range(7))


@pytest.mark.parametrize("seed", range(6))
def test_topk_invariants_with_ties(seed):
    rng = np.random.default_rng(seed)
    nK = int(rng.integers(5, 300))
    S = (rng.integers(0, 7, nK) / 7.0).astype(np.float32)  # many exact ties
    s = int(rng.integers(1, nK + 1))
    idx, _ = O.topk_row(S, s)
    assert len(idx) == s and (np.diff(idx) > 0).all()
    chosen = np.zeros(nK, bool)
    chosen[idx] = True
    if s < nK:
        lo = S[chosen].min()
        hi = S[~chosen].max()
        assert lo >= hi
        # at the boundary value every chosen index precedes every unchosen one
        eq = np.nonzero(S == lo)[0]
        if (S[~chosen] == lo).any():
            assert eq[chosen[eq]].max() < eq[~chosen[eq]].min()


def test_uniform_variant_closed_forms():
    # nK = 8, s = 2: every q' = 2^30 exactly; the draw is the block holding U and the one
    # holding U + 2^32, i.e. {U >> 30, (U >> 30) + 4}
    row, seed, off = 5, 11, 2
    idx, lp = O.plan_row_variant(np.zeros(8, np.float32), 2, seed, off, row, "uniform")
    U = O.plan_uniform(row, seed, off)
    assert idx.tolist() == [U >> 30, (U >> 30) + 4]
    assert np.allclose(lp, np.log(0.25), rtol=0, atol=1e-7)
    # nK = 3, s = 1: lambda = the smallest fp32 with 3 floor(lambda 2^32) >= 2^32; fp32 near
    # 1/3 has spacing 2^-25, so q = ceil(2^32/3) rounded up to a multiple of 2^7, and the
    # last block is trimmed to 2^32 - 2q
    qp, order, _ = O.inclusion_fixed_point(np.ones(3, np.float32), 1)
    q = -(-((1 << 32) // 3 + 1) // 128) * 128
    assert [int(x) for x in qp] == [q, q, (1 << 32) - 2 * q]


def test_no_ipw_variant_is_the_sip_draw_unweighted():
    rng = np.random.default_rng(3)
    S = rng.random(200).astype(np.float32)
    S /= S.sum()
    a = O.plan_row_variant(S, 20, 7, 1, 9, "sip")
    b = O.plan_row_variant(S, 20, 7, 1, 9, "sip_no_ipw")
    assert np.array_equal(a[0], b[0]) and (b[1] == 0).all() and (a[1] <= 0).all()


# ---------------------------------------------------------------- dense attention mass

def test_block_mass_sums_to_one_and_matches_brute_force():
    rng = np.random.default_rng(12)
    N, d, bk = 37, 8, 4          # ragged last block of 1 token
    Qb = rng.standard_normal((5, d))
    Kh = rng.standard_normal((N, d))
    m = O.block_attention_mass(Qb, Kh, bk)
    assert m.shape == (10,) and abs(m.sum() - 1) < 1e-12
    # brute force: per query, per token softmax, summed per block, averaged over queries
    ref = np.zeros(10)
    for q in Qb:
        w = [math.exp(float(q @ k) / math.sqrt(d)) for k in Kh]
        tot = sum(w)
        for t, wt in enumerate(w):
            ref[t // bk] += wt / tot / len(Qb)
    assert np.allclose(m, ref, rtol=1e-12, atol=1e-15)


def test_block_mass_of_identical_keys_is_proportional_to_block_size():
    N, d, bk = 10, 4, 4           # blocks of 4, 4, 2 identical keys
    Kh = np.ones((N, d))
    m = O.block_attention_mass(np.ones((3, d)), Kh, bk)
    assert np.allclose(m, [0.4, 0.4, 0.2], rtol=0, atol=1e-15)
    assert O.mass_topk_row(m, 1).tolist() == [0]   # tie: the lower index
    assert O.mass_topk_row(m, 2).tolist() == [0, 1]
