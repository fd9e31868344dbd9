"""Seeded synthetic inputs for the AB-Attention hot path.

This module only draws random numbers and shapes them; it holds none of the
method's arithmetic (no pooling, clustering, scoring, λ solve, sampling or
attention).  Both the CUDA path and the CPU oracle are fed from here, so the two
see identical bf16 values.

Workloads follow the AB-Attention page (onedev.kr/papers/1521), experiments
paragraph: video DiT layers with 3D raster token order (frame, row, col).  The
real activations of Wan2.1 / HunyuanVideo are not available, so Q and K are a
shared smooth random-Fourier feature of the token position plus noise, which
gives the spatially local, multi-cluster attention structure the selector is
built for; V is Gaussian.  All draws are fp32, then rounded to bf16.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

# Fourier frequency scale (radians per step) along frame, row and column.
FOURIER_SIGMA = (0.35, 0.25, 0.25)


@dataclass(frozen=True)
class Workload:
    """One synthetic layer: shapes plus the plan budget."""

    name: str
    B: int
    H: int
    latent: tuple  # (frames, rows, cols); N = product
    d: int
    kv_block: int
    s: int  # sampled KV blocks per query block
    gen: str  # "gaussian" or "fourier"
    seed: int
    philox_seed: int
    q_block: int = 128
    clusters: int = 8
    kmeans_iters: int = 1
    plan_reuse: int = 1  # attention calls per plan
    perturb_sigma: float = 0.0
    extra: dict = field(default_factory=dict)

    @property
    def N(self) -> int:
        f, r, c = self.latent
        return f * r * c

    @property
    def nQ(self) -> int:
        return -(-self.N // self.q_block)

    @property
    def nK(self) -> int:
        return -(-self.N // self.kv_block)


def budget_blocks(keep_fraction: float, nK: int, kv_block: int, tile: int = 128) -> int:
    """Sampled blocks for a kept fraction, rounded down to whole 128-token tiles.

    s = floor(keep * nK / (tile/bk)) * (tile/bk).  At bk = 4 this gives 2048 of
    18,900 (10.836 % kept, 89.164 % sparse) and 2272 of 29,700 (7.650 % kept),
    the sparsities the experiments paragraph reports.
    """
    per_tile = max(1, tile // kv_block)
    return max(per_tile, int(math.floor(keep_fraction * nK / per_tile)) * per_tile)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, (4, 16, 16), 64, 4, 32, "gaussian", 0, 1),
    "tiny_dense": Workload("tiny_dense", 1, 2, (4, 16, 16), 64, 4, 256, "gaussian", 0, 1),
    "wan13b": Workload("wan13b", 1, 12, (21, 45, 80), 128, 4, 2048, "fourier", 2, 2),
    "wan14b": Workload("wan14b", 1, 40, (21, 45, 80), 128, 4, 2048, "fourier", 3, 3,
                       plan_reuse=4, perturb_sigma=0.05),
    "hunyuan13b": Workload("hunyuan13b", 1, 24, (33, 45, 80), 128, 4, 2272, "fourier", 4, 4),
}
# Granularity sweep at the Wan2.1-1.3B shape: 8192 kept tokens (64 tiles) per query block.
for _bk in (4, 16, 64, 128):
    WORKLOADS[f"sweep_bk{_bk}"] = Workload(
        f"sweep_bk{_bk}", 1, 12, (21, 45, 80), 128, _bk, 8192 // _bk, "fourier", 2, 2)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0xFFFFFFFFFFFF)
    return g


def _head_seed(seed: int, tensor: int, b: int, h: int) -> int:
    # distinct, reproducible stream per (seed, tensor, batch, head)
    return (seed * 1_000_003 + tensor * 7919 + b * 104_729 + h * 31) & 0xFFFFFFFFFFFF


def latent_positions(latent, device="cpu") -> torch.Tensor:
    """[N, 3] fp32 positions (frame, row, col) in raster order."""
    f, r, c = latent
    ff, rr, cc = torch.meshgrid(torch.arange(f, device=device), torch.arange(r, device=device),
                                torch.arange(c, device=device), indexing="ij")
    return torch.stack([ff, rr, cc], -1).reshape(-1, 3).float()


def gaussian_head(N: int, d: int, seed: int, device="cpu") -> torch.Tensor:
    return torch.randn(N, d, generator=_gen(seed, device), device=device, dtype=torch.float32)


def make_qkv(w: Workload, device="cpu", heads=None):
    """Q, K, V as bf16 [B, H, N, d] (or only the listed heads, [B, len(heads), N, d])."""
    heads = list(range(w.H)) if heads is None else list(heads)
    N, d = w.N, w.d
    Q = torch.empty(w.B, len(heads), N, d, dtype=torch.bfloat16, device=device)
    K = torch.empty_like(Q)
    V = torch.empty_like(Q)
    pos = latent_positions(w.latent, device) if w.gen == "fourier" else None
    sig = torch.tensor(FOURIER_SIGMA, device=device)
    for b in range(w.B):
        for hi, h in enumerate(heads):
            if w.gen == "gaussian":
                Q[b, hi] = gaussian_head(N, d, _head_seed(w.seed, 0, b, h), device).bfloat16()
                K[b, hi] = gaussian_head(N, d, _head_seed(w.seed, 1, b, h), device).bfloat16()
            else:
                g = _gen(_head_seed(w.seed, 3, b, h), device)
                W = torch.randn(3, d, generator=g, device=device) * sig[:, None]
                ph = torch.rand(d, generator=g, device=device) * (2 * math.pi)
                phi = math.sqrt(2.0) * torch.cos(pos @ W + ph)
                eq = gaussian_head(N, d, _head_seed(w.seed, 0, b, h), device)
                ek = gaussian_head(N, d, _head_seed(w.seed, 1, b, h), device)
                Q[b, hi] = (0.7 * phi + 0.3 * eq).bfloat16()
                K[b, hi] = (0.7 * phi + 0.3 * ek).bfloat16()
            V[b, hi] = gaussian_head(N, d, _head_seed(w.seed, 2, b, h), device).bfloat16()
    return Q, K, V


def perturb(x: torch.Tensor, sigma: float, seed: int) -> torch.Tensor:
    """x + sigma * N(0,1), rounded to bf16 (the per-step drift between plan refreshes)."""
    e = torch.randn(x.shape, generator=_gen(seed, x.device), device=x.device, dtype=torch.float32)
    return (x.float() + sigma * e).bfloat16()


def random_scores(rows: int, nK: int, seed: int, device="cpu", sigma: float = 2.0,
                  zero_frac: float = 0.0) -> torch.Tensor:
    """[rows, nK] fp32 nonnegative rows with unit sum and a heavy (log-normal) head.

    A stand-in score matrix for planner tests: a few blocks carry most of the
    mass (so some inclusion probabilities saturate at 1) and the rest form a long
    tail.  Optionally a fraction of entries is exactly zero.
    """
    g = _gen(seed, device)
    x = torch.exp(sigma * torch.randn(rows, nK, generator=g, device=device))
    if zero_frac > 0:
        x = torch.where(torch.rand(rows, nK, generator=g, device=device) < zero_frac,
                        torch.zeros_like(x), x)
    return (x / x.sum(1, keepdim=True)).float()


def random_plan(rows: int, nK: int, s: int, seed: int, device="cpu"):
    """A synthetic plan: per row s distinct ascending block indices and log-probabilities.

    logπ is drawn in [ln 0.02, 0] with about a quarter of entries exactly 0
    (saturated blocks).  Used to exercise the attention kernel at full size on
    rows the oracle cannot plan itself in reasonable time.
    """
    g = _gen(seed, device)
    idx = torch.empty(rows, s, dtype=torch.int32, device=device)
    chunk = max(1, (1 << 26) // max(nK, 1))
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        keys = torch.rand(r1 - r0, nK, generator=g, device=device)
        idx[r0:r1] = torch.topk(keys, s, dim=1).indices.sort(dim=1).values.int()
    u = torch.rand(rows, s, generator=g, device=device)
    logpi = torch.where(u < 0.25, torch.zeros_like(u), math.log(0.02) * torch.rand(
        rows, s, generator=g, device=device))
    return idx, logpi.float()
