"""Plain fp64 CPU oracle for the AB-Attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA library and imports nothing from the package.

Every step follows the AB-Attention page (onedev.kr/papers/1521):

* [IBCS]   section "how it differs" (무엇과 다른가): 128-token query blocks,
           4-token KV blocks, one k-means iteration into 8 query clusters per
           query block, cluster centroids and query shares, block score = the
           share-weighted softmax mass of the centroids over pooled keys.
* [SIP]    section "how to use" (어떻게 쓰나): π_ij = min(1, λ_i S_ij) with
           Σ_j π_ij = s; π = 1 blocks always kept; systematic sampling of exactly
           s distinct blocks shared by the query block; 1/π weighting of
           numerator and denominator ≡ a −log π logit shift.
* [KERNEL] section "premises & limits" (전제와 한계), first paragraph: sampled
           small blocks gathered by index into full tiles; −log π shift, online
           softmax and value accumulation in one pass; no token reordering.
* [ABL]    ablation paragraph: position-based 16-query segment means (used here
           as the k-means initialisation, and alone when kmeans_iters = 0), and
           the selection rules SIP is compared against: deterministic top-k,
           sampling without inverse-probability weighting, uniform sampling.

Where the page is silent the oracle takes these readings (the same ones the
CUDA path implements):

  R1  k-means starts from the 8 contiguous segment means of the valid rows
      (segment c = rows [floor(c n/8), floor((c+1) n/8))), computed in fp64.
  R2  one iteration = one assignment (squared Euclidean, fp64, ties to the
      lowest cluster) + one update (fp64 member means).
  R3  share w_c = |members| / n_valid; an empty cluster gets w = 0 and a zero
      centroid.
  R4  pooled key = mean of the block's valid keys (fp64 sum / count).
  R5  centroids and pooled keys are rounded once, to bf16 (round to nearest
      even), from the exact fp64 means; logits = <c, k̄>/sqrt(d); softmax over all
      KV blocks of the head; S in fp32.
  R6  λ and π in 2^-32 fixed point: for an fp32 λ, x_j = fl32(λ S_j),
      q_j = 2^32 if x_j >= 1 else floor(x_j 2^32); F(λ) = Σ q_j.  λ* is the
      smallest positive fp32 with F(λ*) >= s 2^32 (bisection over the bit
      patterns).  Blocks are laid out saturated-first (ascending j), then the
      rest (ascending j); the prefix is capped at s 2^32 so Σ q' = s 2^32
      exactly.  π' = q'/2^32 is the exact inclusion probability; log π' in fp64,
      stored as fp32.  If fewer than s blocks have S > 0, every positive block
      and the lowest-index zero blocks are taken with π = 1.
  R7  systematic sampling on the lattice U + k 2^32 (k = 0..s-1), U = word 0 of
      Philox4x32-10 with key (seed_lo, seed_hi) and counter
      (row, offset_lo, offset_hi, 0), row = (b H + h) nQ + i.
  R8  attention logits z = q.k/sqrt(d) - log π_j over the valid tokens of the
      sampled blocks; softmax and value sum in fp64.
  R9  planner variants: top-k = the s largest S_j (ties to the lower j; scores
      ranked by the order-preserving key of their fp32 bit pattern, so +0 ranks
      above -0 and NaN below every number), log π = 0; "no IPW" = the SIP draw
      with log π = 0; "uniform" = the SIP fixed point and draw on a constant
      score row (π_j = s/nK up to the 2^-32 fixed point and the trimmed tail).
"""

from __future__ import annotations

import math

import numpy as np

TWO32 = 1 << 32

# --------------------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even) of fp64 values
# --------------------------------------------------------------------------------------


def bf16_round(x) -> np.ndarray:
    """Nearest bf16 value of each fp64 entry (ties to even), returned as fp64.

    Done on the fp64 bit pattern: bf16 keeps 7 of the 52 fraction bits, so the
    low 45 bits are rounded away with the usual add-half-minus-one-plus-lsb
    trick.  Magnitudes below the smallest normal bf16 (2^-126) are rounded on
    the subnormal grid 2^-133; results beyond the largest finite bf16 become inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    ax = np.abs(x)
    normal = ax >= 2.0 ** -126
    u = x.view(np.uint64)
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    r = (u + (np.uint64((1 << 44) - 1) + lsb)) & ~np.uint64((1 << 45) - 1)
    rv = r.view(np.float64)
    out[normal] = rv[normal]
    sub = ~normal
    out[sub] = np.rint(x[sub] / 2.0 ** -133) * 2.0 ** -133  # rint: ties to even
    big = np.abs(out) >= 2.0 ** 128
    out[big] = np.copysign(np.inf, x[big])
    nan = np.isnan(x)
    out[nan] = np.nan
    return out


# --------------------------------------------------------------------------------------
# IBCS: pooled keys, intra-block k-means, block scores   ([IBCS], R1-R5)
# --------------------------------------------------------------------------------------


def pool_keys(K: np.ndarray, kv_block: int) -> np.ndarray:
    """Pooled key per KV block: bf16(mean of the block's valid keys).  K: [N, d] fp64."""
    N, d = K.shape
    nK = -(-N // kv_block)
    out = np.empty((nK, d))
    for j in range(nK):
        blk = K[j * kv_block: min(N, (j + 1) * kv_block)]
        out[j] = blk.sum(0) / blk.shape[0]
    return bf16_round(out)


def segment_bounds(n: int, C: int):
    return [(c * n // C, (c + 1) * n // C) for c in range(C)]


def kmeans_block(Qb: np.ndarray, C: int = 8, iters: int = 1):
    """One query block: returns (centroids bf16-as-fp64 [C, d], w [C], labels [n], gap [n]).

    Qb: [n, d] fp64 (the bf16 query rows).  Initial centroids are the C
    contiguous segment means (R1); each iteration assigns every query to the
    nearest centroid in squared Euclidean distance (ties to the lowest index)
    and replaces each centroid by the mean of its members (R2).  gap is the
    relative distance gap (d2 - d1) / d2 between the best (d1) and second-best
    (d2) live centroid of the last assignment; clusters emptied by an earlier
    iteration take no part; inf when there is no assignment or only one live
    cluster; 0 on an exact tie.
    """
    n, d = Qb.shape
    cent = np.zeros((C, d))
    alive = np.zeros(C, dtype=bool)
    counts = np.zeros(C, dtype=np.int64)
    for c, (a, b) in enumerate(segment_bounds(n, C)):
        if b > a:
            cent[c] = Qb[a:b].sum(0) / (b - a)
            alive[c] = True
            counts[c] = b - a
    labels = np.repeat(np.arange(C), [b - a for a, b in segment_bounds(n, C)])
    gap = np.full(n, np.inf)
    for _ in range(iters):
        dist = ((Qb[:, None, :] - cent[None, :, :]) ** 2).sum(-1)  # [n, C]
        dist[:, ~alive] = np.inf
        labels = np.argmin(dist, axis=1)  # first minimum: lowest index on ties
        srt = np.sort(dist, axis=1)
        with np.errstate(invalid="ignore", divide="ignore"):
            gap = (srt[:, 1] - srt[:, 0]) / np.maximum(srt[:, 1], 1e-300)
        gap[np.isinf(srt[:, 1])] = np.inf  # one live cluster: no runner-up, no near-tie
        new = np.zeros((C, d))
        counts = np.bincount(labels, minlength=C)
        for c in range(C):
            if counts[c]:
                new[c] = Qb[labels == c].sum(0) / counts[c]
            else:
                new[c] = cent[c]
        cent = new
        alive = counts > 0
    w = counts / n
    out = np.where(alive[:, None], bf16_round(cent), 0.0)
    w = np.where(alive, w, 0.0)
    return out, w, labels, gap


def block_scores(cent: np.ndarray, w: np.ndarray, Kp: np.ndarray) -> np.ndarray:
    """S_j = Σ_c w_c softmax_j(<cent_c, Kp_j>/sqrt(d)) over all KV blocks, fp64 (R5)."""
    d = Kp.shape[1]
    logits = (cent @ Kp.T) / math.sqrt(d)  # [C, nK]
    logits -= logits.max(1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(1, keepdims=True)
    return (w[:, None] * p).sum(0)


def select_head(Qh: np.ndarray, Kh: np.ndarray, q_block=128, kv_block=4, C=8, iters=1,
                rows=None, debug=False):
    """IBCS for one (b, h): S [len(rows), nK] as fp32 (fp64 values rounded once).

    Qh, Kh: [N, d] fp64 holding the bf16 inputs.  rows: query-block indices
    (default all).  With debug=True also returns per-row (cent, w, labels, gap).
    """
    N = Qh.shape[0]
    nQ = -(-N // q_block)
    rows = range(nQ) if rows is None else rows
    Kp = pool_keys(Kh, kv_block)
    S, dbg = [], []
    for i in rows:
        Qb = Qh[i * q_block: min(N, (i + 1) * q_block)]
        cent, w, labels, gap = kmeans_block(Qb, C, iters)
        S.append(block_scores(cent, w, Kp))
        dbg.append((cent, w, labels, gap))
    S = np.array(S).astype(np.float32)
    return (S, dbg, Kp) if debug else S


def scores_from_labels(Qb: np.ndarray, labels: np.ndarray, Kp: np.ndarray, C: int = 8):
    """S row recomputed from given cluster labels (for near-tie excusal in tests)."""
    n, d = Qb.shape
    cent = np.zeros((C, d))
    counts = np.bincount(labels, minlength=C)
    for c in range(C):
        if counts[c]:
            cent[c] = bf16_round(Qb[labels == c].sum(0) / counts[c])
    return block_scores(cent, counts / n, Kp).astype(np.float32)


# --------------------------------------------------------------------------------------
# Philox4x32-10 (Salmon, Moraes, Dror, Shaw: "Parallel random numbers: as easy as
# 1, 2, 3", SC'11), written generically over the word size
# --------------------------------------------------------------------------------------

PHILOX4x32 = dict(w=32, M0=0xD2511F53, M1=0xCD9E8D57, W0=0x9E3779B9, W1=0xBB67AE85)


def philox4(ctr, key, rounds=10, w=32, M0=0, M1=0, W0=0, W1=0):
    """Philox4xW-R block function on Python ints: 4-word counter, 2-word key."""
    m = (1 << w) - 1
    x0, x1, x2, x3 = (int(v) & m for v in ctr)
    k0, k1 = (int(v) & m for v in key)
    for r in range(rounds):
        if r:
            k0, k1 = (k0 + W0) & m, (k1 + W1) & m
        p0, p1 = M0 * x0, M1 * x2
        x0, x1, x2, x3 = ((p1 >> w) ^ x1 ^ k0) & m, p1 & m, ((p0 >> w) ^ x3 ^ k1) & m, p0 & m
    return x0, x1, x2, x3


def philox4x32_10(ctr, key):
    return philox4(ctr, key, 10, **PHILOX4x32)


def plan_uniform(row: int, seed: int, offset: int) -> int:
    """U in [0, 2^32) for one plan row (R7)."""
    return philox4x32_10((row & 0xFFFFFFFF, offset & 0xFFFFFFFF, (offset >> 32) & 0xFFFFFFFF, 0),
                         (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))[0]


# --------------------------------------------------------------------------------------
# SIP: λ, fixed-point π, systematic sampling   ([SIP], R6, R7)
# --------------------------------------------------------------------------------------


def f32_from_bits(b: int) -> np.float32:
    return np.array([b], dtype=np.uint32).view(np.float32)[0]


def fixed_point_q(lam_bits: int, S: np.ndarray) -> np.ndarray:
    """q_j(λ) in units of 2^-32 (uint64): 2^32 if fl32(λ S_j) >= 1, else floor(fl32(λ S_j) 2^32)."""
    lam = f32_from_bits(lam_bits)
    S = np.asarray(S, dtype=np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        x = (np.float32(lam) * S).astype(np.float32)  # one fp32 rounding per product
    pos = S > 0
    sat = pos & (x >= 1)
    frac = np.where(pos & ~sat, x, 0).astype(np.float64) * TWO32
    q = np.floor(frac).astype(np.uint64)
    q[sat] = TWO32
    return q


def solve_lambda(S: np.ndarray, s: int):
    """Smallest positive fp32 λ (as bit pattern) with Σ q_j(λ) >= s 2^32, or None.

    None means fewer than s blocks have S > 0 (then no λ reaches the budget).
    """
    target = s * TWO32
    lo, hi = 0, 0x7F800000  # F(0) = 0 < target; hi = +inf
    if int(fixed_point_q(hi, S).sum()) < target:
        return None
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if int(fixed_point_q(mid, S).sum()) >= target:
            hi = mid
        else:
            lo = mid
    return hi


def inclusion_fixed_point(S: np.ndarray, s: int):
    """Exact inclusion probabilities q' (uint64, units of 2^-32) and the layout order.

    Returns (qp, order, lam_bits): qp[j] = 2^32 π'_j with Σ qp = s 2^32; order is
    the cumulative layout (saturated blocks ascending, then the rest ascending).
    """
    S = np.asarray(S, dtype=np.float32)
    nK = S.shape[0]
    lam_bits = solve_lambda(S, s)
    if lam_bits is None:
        pos = np.flatnonzero(S > 0)
        zeros = np.flatnonzero(~(S > 0))[: s - len(pos)]
        qp = np.zeros(nK, dtype=np.uint64)
        qp[pos] = TWO32
        qp[zeros] = TWO32
        sat = qp == TWO32
        order = np.concatenate([np.flatnonzero(sat), np.flatnonzero(~sat)])
        return qp, order, None
    q = fixed_point_q(lam_bits, S)
    sat = q == TWO32
    order = np.concatenate([np.flatnonzero(sat), np.flatnonzero(~sat)])
    target = s * TWO32
    Q = np.cumsum(q[order], dtype=np.uint64)  # exact: the total is below nK * 2^32 < 2^64
    Qc = np.minimum(Q, np.uint64(target))
    prev = np.concatenate([np.zeros(1, dtype=np.uint64), Qc[:-1]])
    qp = np.zeros(nK, dtype=np.uint64)
    qp[order] = Qc - prev
    return qp, order, lam_bits


def systematic_sample(qp: np.ndarray, order: np.ndarray, U: int, s: int) -> np.ndarray:
    """Madow systematic πps sample on the integer lattice U + k 2^32, k = 0..s-1.

    Block j occupies [start_j, end_j) of length qp[j] in the layout order; it is
    selected iff a lattice point falls in that interval.  Returns ascending j.
    """
    def M(x):  # number of lattice points below x
        return 0 if x <= U else min(s, (x - U - 1) // TWO32 + 1)

    pos = 0
    chosen = []
    for j in order:
        end = pos + int(qp[j])
        if M(end) > M(pos):
            chosen.append(int(j))
        pos = end
    return np.array(sorted(chosen), dtype=np.int64)


def plan_row(S: np.ndarray, s: int, seed: int, offset: int, row: int):
    """SIP for one query block: (idx ascending int32 [s], logπ fp32 [s], qp uint64 [nK])."""
    qp, order, _ = inclusion_fixed_point(S, s)
    U = plan_uniform(row, seed, offset)
    idx = systematic_sample(qp, order, U, s)
    logpi = np.array([math.log(int(qp[j]) / TWO32) for j in idx], dtype=np.float64)
    return idx.astype(np.int32), logpi.astype(np.float32), qp


def score_key(S: np.ndarray) -> np.ndarray:
    """Order-preserving uint32 key of fp32 scores (R9): larger score, larger key; NaN -> 0."""
    b = np.asarray(S, dtype=np.float32).view(np.uint32).astype(np.uint64)
    neg = (b >> 31) == 1
    key = np.where(neg, (~b) & 0xFFFFFFFF, b | 0x80000000)
    key = np.where(np.isnan(np.asarray(S, dtype=np.float32)), 0, key)
    return key.astype(np.uint64)


def topk_row(S: np.ndarray, s: int):
    """[ABL] deterministic top-k: the s largest scores, ties to the lower index (R9).

    Returns (idx ascending int32 [s], logπ = 0 fp32 [s]).  A plain sort of
    (-key, index) pairs.
    """
    key = score_key(S)
    ranked = sorted(range(len(key)), key=lambda j: (-int(key[j]), j))
    idx = np.array(sorted(ranked[:s]), dtype=np.int32)
    return idx, np.zeros(s, dtype=np.float32)


def plan_row_variant(S: np.ndarray, s: int, seed: int, offset: int, row: int, mode: str):
    """One query block's plan under a planner variant (R9): "sip", "sip_no_ipw",
    "uniform" or "topk".  Returns (idx ascending int32 [s], logπ fp32 [s])."""
    if mode == "sip":
        idx, lp, _ = plan_row(S, s, seed, offset, row)
        return idx, lp
    if mode == "sip_no_ipw":
        idx, _, _ = plan_row(S, s, seed, offset, row)
        return idx, np.zeros(s, dtype=np.float32)
    if mode == "uniform":
        idx, lp, _ = plan_row(np.ones(len(S), dtype=np.float32), s, seed, offset, row)
        return idx, lp
    if mode == "topk":
        return topk_row(S, s)
    raise ValueError(mode)


def sample_row(pi: np.ndarray, s: int, seed: int, offset: int, row: int):
    """Sampling given target inclusion probabilities π (fp32, Σ ≈ s).

    The probabilities are re-solved through the same fixed-point λ step (π is
    used as the score vector), so the draw has exactly s blocks and Σ π' = s
    holds in 2^-32 units; when the given π already sum to s the rescale factor is
    1 to within fp32 rounding.
    """
    return plan_row(np.asarray(pi, dtype=np.float32), s, seed, offset, row)


# --------------------------------------------------------------------------------------
# Attention   ([SIP] logit shift, [KERNEL], R8)
# --------------------------------------------------------------------------------------


def attn_block(Qb: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, idx, logpi, kv_block: int):
    """O for one query block over its sampled KV blocks with the −log π shift, fp64.

    Qb: [n, d]; Kh, Vh: [N, d]; idx, logpi: [s].  Tokens beyond N in the last
    block are skipped.
    """
    N, d = Kh.shape
    toks, shift = [], []
    for j, lp in zip(np.asarray(idx), np.asarray(logpi, dtype=np.float64)):
        t = np.arange(int(j) * kv_block, min(N, (int(j) + 1) * kv_block))
        toks.append(t)
        shift.append(np.full(t.shape, lp))
    toks = np.concatenate(toks)
    shift = np.concatenate(shift)
    z = (Qb @ Kh[toks].T) / math.sqrt(d) - shift[None, :]
    z -= z.max(1, keepdims=True)
    p = np.exp(z)
    return (p @ Vh[toks]) / p.sum(1, keepdims=True)


def attn_head(Qh, Kh, Vh, idx_rows, logpi_rows, rows, q_block=128, kv_block=4):
    """O rows for the listed query blocks of one head; returns a dict i -> [n, d]."""
    N = Qh.shape[0]
    return {i: attn_block(Qh[i * q_block: min(N, (i + 1) * q_block)], Kh, Vh, idx_rows[k],
                          logpi_rows[k], kv_block) for k, i in enumerate(rows)}


def dense_attention(Qr: np.ndarray, Kh: np.ndarray, Vh: np.ndarray) -> np.ndarray:
    """Textbook softmax(Q K^T / sqrt(d)) V in fp64 for the given query rows."""
    z = (Qr @ Kh.T) / math.sqrt(Kh.shape[1])
    z -= z.max(1, keepdims=True)
    p = np.exp(z)
    return (p @ Vh) / p.sum(1, keepdims=True)


def block_attention_mass(Qb: np.ndarray, Kh: np.ndarray, kv_block: int) -> np.ndarray:
    """Dense softmax mass of each KV block, averaged over the query block's rows, fp64.

    m_j = (1/n) Σ_q Σ_{t in block j} softmax_t(q.k/sqrt(d)); Σ_j m_j = 1.  The quantity
    whose top-s the selector tries to find ([IBCS] "which KV blocks matter"; the ablation
    paragraph's attention-mass figures).  Measurement only.
    """
    N, d = Kh.shape
    z = (Qb @ Kh.T) / math.sqrt(d)
    z -= z.max(1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(1, keepdims=True)
    nK = -(-N // kv_block)
    padded = np.zeros((Qb.shape[0], nK * kv_block))
    padded[:, :N] = p
    return padded.reshape(Qb.shape[0], nK, kv_block).sum(2).mean(0)


def mass_topk_row(mass: np.ndarray, s: int) -> np.ndarray:
    """The s blocks of largest dense attention mass (ties to the lower index), ascending:
    the oracle top-k the selector's choices are measured against."""
    ranked = sorted(range(len(mass)), key=lambda j: (-float(mass[j]), j))
    return np.array(sorted(ranked[:s]), dtype=np.int32)


def ht_estimates(Qb, Kh, Vh, idx, qp, kv_block):
    """Horvitz–Thompson numerator [n, d] and denominator [n] of one sample, fp64.

    Each sampled block's unnormalised attention terms e^{q.k/sqrt(d)} v and
    e^{q.k/sqrt(d)} are weighted by 1/π'_j ([SIP]); max-shifted by the dense row
    max m so the dense values are Σ_t e^{z_t - m} v_t and Σ_t e^{z_t - m}.
    """
    N, d = Kh.shape
    zfull = (Qb @ Kh.T) / math.sqrt(d)
    m = zfull.max(1, keepdims=True)
    num = np.zeros((Qb.shape[0], Vh.shape[1]))
    den = np.zeros(Qb.shape[0])
    for j in np.asarray(idx):
        t = np.arange(int(j) * kv_block, min(N, (int(j) + 1) * kv_block))
        e = np.exp(zfull[:, t] - m)
        pi = int(qp[j]) / TWO32
        num += (e @ Vh[t]) / pi
        den += e.sum(1) / pi
    return num, den
