"""The denoising-loop attention schedule of the AB-Attention page (main experiments).

The first transformer block and the first 10 denoising steps keep dense attention; after
that every block's sampling plan is rebuilt every 4 steps and reused in between, while the
attention itself runs every step on the current activations (AB-Attention page,
onedev.kr/papers/1521, main-experiments paragraph; plan reuse in the "how to use"
section).  A rebuilt plan draws with Philox offset = the refresh index (0, 1, 2, ...) and
seed = base seed + block index, so successive refreshes and different blocks draw
independently.

Host-side bookkeeping only: every computation is a library call (ab_attn_dense, ab_select,
ab_plan, ab_attn) on the caller's CUDA stream.
"""

from __future__ import annotations

DENSE = "dense"
REFRESH = "refresh"
REUSE = "reuse"


def schedule_mode(block: int, step: int, dense_steps: int = 10, refresh: int = 4) -> str:
    """What block `block` does at denoising step `step`: DENSE, REFRESH (rebuild the plan,
    then sparse attention) or REUSE (sparse attention with the block's last plan)."""
    if block == 0 or step < dense_steps:
        return DENSE
    return REFRESH if (step - dense_steps) % refresh == 0 else REUSE


def refresh_index(step: int, dense_steps: int = 10, refresh: int = 4) -> int:
    """Index of the plan in use at `step` (0 for the first sparse step's plan)."""
    return (step - dense_steps) // refresh


class SparseAttentionSchedule:
    """Attention of a DiT with `n_blocks` transformer blocks over the denoising steps.

    One instance holds, per sparse block, the current plan (idx int32 and log pi fp32,
    [B*H*nQ, s] each) and one shared score buffer and selector workspace.
    """

    def __init__(self, B: int, H: int, N: int, d: int, n_blocks: int, s: int, kv_block: int = 4,
                 clusters: int = 8, kmeans_iters: int = 1, dense_steps: int = 10, refresh: int = 4,
                 seed: int = 0, device="cuda"):
        import torch

        from . import ab_workspace_bytes, params

        self.p = params(B, H, N, d, kv_block, clusters, kmeans_iters)
        self.s, self.seed = s, seed
        self.dense_steps, self.refresh = dense_steps, refresh
        nQ = (N + 127) // 128
        nK = (N + kv_block - 1) // kv_block
        rows = B * H * nQ
        self.S = torch.empty(B, H, nQ, nK, device=device)
        self.ws = torch.empty(ab_workspace_bytes(self.p), dtype=torch.uint8, device=device)
        self.idx = [torch.empty(rows, s, dtype=torch.int32, device=device) if b else None
                    for b in range(n_blocks)]
        self.logpi = [torch.empty(rows, s, device=device) if b else None for b in range(n_blocks)]
        self.calls = {DENSE: 0, REFRESH: 0, REUSE: 0}

    def attention(self, block: int, step: int, Q, K, V, O, stream=None) -> str:
        """O = attention of block `block` at step `step` (Q, K, V, O bf16 [B, H, N, d])."""
        from . import ab_attn, ab_attn_dense, ab_plan, ab_select

        mode = schedule_mode(block, step, self.dense_steps, self.refresh)
        if mode == DENSE:
            ab_attn_dense(self.p, Q, K, V, O, stream)
        else:
            if mode == REFRESH:
                ab_select(self.p, Q, K, self.S, self.ws, stream)
                ab_plan(self.p, self.S, self.s, self.seed + block,
                        refresh_index(step, self.dense_steps, self.refresh),
                        self.idx[block], self.logpi[block], stream)
            ab_attn(self.p, Q, K, V, self.idx[block], self.logpi[block], self.s, O, stream)
        self.calls[mode] += 1
        return mode
