"""Ablation measurement on synthetic inputs (measurement tool; uses the oracle).

The AB-Attention page (onedev.kr/papers/1521) compares its selector and planner with
simpler rules: position-based segment means instead of k-means clusters, deterministic
top-k instead of sampling, sampling without inverse-probability weights, uniform
sampling.  This script runs each rule through the library on one head of a synthetic
workload and measures, on a fixed sample of query blocks, against fp64 dense attention
(oracle):

  err   rel-L2 of O against dense attention, ||O - O_dense||_F / ||O_dense||_F
  mass  dense attention mass of the kept blocks (oracle block mass, averaged over the
        block's queries and then over the sampled blocks)

plus the oracle top-k by dense mass (the best any top-s block choice can capture).
The page's own figures come from real video activations and are not reproduced here.

    python tests/ablation_report.py [--workload wan13b] [--blocks 16] [--head 0] [--json PATH]
"""

from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)

VARIANTS = [  # (name, k-means iterations of the selector, planner mode)
    ("sip", 1, "sip"),
    ("sip_segment_means", 0, "sip"),
    ("sip_no_ipw", 1, "sip_no_ipw"),
    ("uniform", 1, "uniform"),
    ("topk_ibcs", 1, "topk"),
    ("topk_segment_means", 0, "topk"),
]


def sample_blocks(nQ: int, k: int):
    """k query blocks spread over the head, the first and the last included."""
    if k >= nQ:
        return list(range(nQ))
    return sorted({int(round(x)) for x in np.linspace(0, nQ - 1, k)})


def run_ablation(workload: str = "wan13b", blocks: int = 16, head: int = 0, seed_offset: int = 0):
    import torch

    import block_sparse_attention_ibcs_b200 as ab
    from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv
    from oracle import abattn_oracle as O

    w = WORKLOADS[workload]
    Q, K, V = make_qkv(w, device="cuda", heads=[head])
    N, d, bk, s = w.N, w.d, w.kv_block, w.s
    nQ = (N + 127) // 128
    nK = (N + bk - 1) // bk

    # ---- GPU: scores (k-means 1 and 0 iterations), plans, attention
    outs, plans = {}, {}
    scores = {}
    for iters in (1, 0):
        p = ab.params(1, 1, N, d, bk, w.clusters, iters)
        S = torch.empty(1, 1, nQ, nK, device="cuda")
        ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
        ab.ab_select(p, Q, K, S, ws)
        scores[iters] = S
    p = ab.params(1, 1, N, d, bk, w.clusters, 1)
    for name, iters, mode in VARIANTS:
        idx = torch.empty(nQ, s, dtype=torch.int32, device="cuda")
        lp = torch.empty(nQ, s, device="cuda")
        ab.ab_plan_variant(p, scores[iters], s, w.philox_seed, seed_offset, mode, idx, lp)
        Od = torch.empty_like(Q)
        ab.ab_attn(p, Q, K, V, idx, lp, s, Od)
        plans[name] = (idx.cpu().numpy(), lp.cpu().numpy())
        outs[name] = Od[0, 0].float().cpu().numpy()
    assert ab.ab_get_status() == 0

    # ---- oracle: dense attention, block mass, oracle top-k by mass
    qh = Q[0, 0].double().cpu().numpy()
    kh = K[0, 0].double().cpu().numpy()
    vh = V[0, 0].double().cpu().numpy()
    rows = sample_blocks(nQ, blocks)
    acc = {name: [0.0, 0.0, 0.0] for name, _, _ in VARIANTS}  # err^2, ref^2, mass
    acc["topk_oracle_mass"] = [0.0, 0.0, 0.0]
    t0 = time.time()
    for i in rows:
        sl = slice(i * 128, min(N, (i + 1) * 128))
        Qb = qh[sl]
        dense = O.dense_attention(Qb, kh, vh)
        mass = O.block_attention_mass(Qb, kh, bk)
        ref2 = float((dense ** 2).sum())
        for name, _, _ in VARIANTS:
            e = outs[name][sl] - dense
            acc[name][0] += float((e ** 2).sum())
            acc[name][1] += ref2
            acc[name][2] += float(mass[plans[name][0][i]].sum())
        oidx = O.mass_topk_row(mass, s)
        o_or = O.attn_block(Qb, kh, vh, oidx, np.zeros(s), bk)
        acc["topk_oracle_mass"][0] += float(((o_or - dense) ** 2).sum())
        acc["topk_oracle_mass"][1] += ref2
        acc["topk_oracle_mass"][2] += float(mass[oidx].sum())
    res = {
        name: {"rel_l2_err": (a[0] / a[1]) ** 0.5, "mass_captured": a[2] / len(rows)}
        for name, a in acc.items()
    }
    return {
        "workload": workload, "head": head, "query_blocks": rows, "s": s, "nK": nK,
        "kept_fraction": s / nK, "oracle_seconds": round(time.time() - t0, 1), "variants": res,
    }


def run_granularity_sweep(blocks: int = 32):
    """Selection granularity at a fixed budget of 8192 kept tokens per query block
    (Wan2.1-1.3B shape, KV block 4, 16, 64, 128): rel-L2 error of the SIP output against
    fp64 dense attention on head 0, `blocks` fixed query blocks (first and last included).
    The page's ablation reports quality improving steadily as the selected blocks shrink
    toward 4 tokens, with the packing keeping the tensor-core work unchanged."""
    import torch

    import block_sparse_attention_ibcs_b200 as ab
    from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv
    from oracle import abattn_oracle as O

    base = WORKLOADS["sweep_bk4"]
    Q, K, V = make_qkv(base, device="cuda", heads=[0])
    N, d = base.N, base.d
    nQ = (N + 127) // 128
    rows_q = sample_blocks(nQ, blocks)
    rows = np.concatenate([np.arange(i * 128, min(N, (i + 1) * 128)) for i in rows_q])
    q0, k0, v0 = (t[0, 0].double().cpu().numpy() for t in (Q, K, V))
    dense = O.dense_attention(q0[rows], k0, v0)
    cases = []
    for bk in (4, 16, 64, 128):
        w = WORKLOADS[f"sweep_bk{bk}"]
        p = ab.params(1, 1, N, d, bk)
        nK = (N + bk - 1) // bk
        S = torch.empty(1, 1, nQ, nK, device="cuda")
        ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
        idx = torch.empty(nQ, w.s, dtype=torch.int32, device="cuda")
        lp = torch.empty(nQ, w.s, device="cuda")
        Od = torch.empty_like(Q)
        ab.ab_select(p, Q, K, S, ws)
        ab.ab_plan(p, S, w.s, w.philox_seed, 0, idx, lp)
        ab.ab_attn(p, Q, K, V, idx, lp, w.s, Od)
        assert ab.ab_get_status() == 0
        got = Od[0, 0].double().cpu().numpy()[rows]
        cases.append({"kv_block": bk, "s": w.s, "tiles_per_query_block": -(-w.s * bk // 128),
                      "rel_l2_vs_dense_fp64": float(np.linalg.norm(got - dense) / np.linalg.norm(dense))})
    return {"workload": "sweep (Wan2.1-1.3B shape, head 0)", "query_blocks": rows_q, "cases": cases}


def markdown(rep) -> str:
    lines = [f"workload {rep['workload']}, head {rep['head']}, {len(rep['query_blocks'])} query "
             f"blocks, s = {rep['s']} of {rep['nK']} blocks ({100 * rep['kept_fraction']:.2f} %)",
             "", "| variant | rel-L2 error vs dense | dense attention mass kept |", "|---|---|---|"]
    for name, v in rep["variants"].items():
        lines.append(f"| {name} | {v['rel_l2_err']:.4f} | {100 * v['mass_captured']:.2f} % |")
    return "\n".join(lines)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="wan13b")
    ap.add_argument("--blocks", type=int, default=16)
    ap.add_argument("--head", type=int, default=0)
    ap.add_argument("--json", default=None)
    ap.add_argument("--sweep", action="store_true",
                    help="granularity sweep (KV block 4..128 at 8192 kept tokens) instead")
    a = ap.parse_args()
    if a.sweep:
        rep = run_granularity_sweep(max(a.blocks, 32))
        for c in rep["cases"]:
            print(f"kv_block {c['kv_block']:4d}  s {c['s']:5d}  tiles {c['tiles_per_query_block']}  "
                  f"rel-L2 vs dense {c['rel_l2_vs_dense_fp64']:.5f}")
    else:
        rep = run_ablation(a.workload, a.blocks, a.head)
        print(markdown(rep))
    if a.json:
        with open(a.json, "w") as f:
            json.dump(rep, f, indent=1)


if __name__ == "__main__":
    main()
