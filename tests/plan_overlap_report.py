"""Plan overlap between neighbouring query blocks (measurement tool; uses the oracle, CPU only).

The packed attention gathers every query block's sampled KV blocks on its own; two query
blocks whose plans share blocks gather those twice.  This script measures, on one head of
a synthetic workload, how much the SIP plans (AB-Attention page, onedev.kr/papers/1521,
section "how to use") of query blocks i and i+1 have in common:

  shared      |idx_i ∩ idx_{i+1}| / s
  saturated   blocks with pi = 1 in plan i, / s
  shared_sat  saturated blocks of plan i that plan i+1 also holds, / s

over a fixed sample of query-block pairs, with the oracle's IBCS scores and planner (the
library produces the same plans bit for bit).  It sizes how much of the gather two CTAs of
a cluster could share.

    python tests/plan_overlap_report.py [--workload wan13b] [--head 0] [--pairs 24] [--json PATH]
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="wan13b")
    ap.add_argument("--head", type=int, default=0)
    ap.add_argument("--pairs", type=int, default=24, help="query-block pairs, spread evenly")
    ap.add_argument("--json", default=None)
    args = ap.parse_args(argv)

    from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv
    from oracle import abattn_oracle as O

    w = WORKLOADS[args.workload]
    t0 = time.time()
    Q, K, _ = make_qkv(w, heads=[args.head])
    Qh, Kh = Q[0, 0].double().numpy(), K[0, 0].double().numpy()
    firsts = sorted(set(np.linspace(0, w.nQ - 2, args.pairs).round().astype(int).tolist()))
    rows = sorted(set(firsts) | {i + 1 for i in firsts})
    S = O.select_head(Qh, Kh, 128, w.kv_block, w.clusters, w.kmeans_iters, rows=rows)
    S = dict(zip(rows, S))
    plans = {}
    for i in rows:
        row = (args.head * w.nQ) + i  # b = 0
        idx, _, qp = O.plan_row(S[i], w.s, w.philox_seed, 0, row)
        plans[i] = (set(idx.tolist()), {j for j in idx.tolist() if int(qp[j]) == O.TWO32})
    per = []
    for i in firsts:
        a, sat_a = plans[i]
        b, _ = plans[i + 1]
        per.append({"qb": i, "shared": len(a & b) / w.s, "saturated": len(sat_a) / w.s,
                    "shared_sat": len(sat_a & b) / w.s})
    out = {
        "workload": args.workload, "head": args.head, "s": w.s, "nK": w.nK, "pairs": len(per),
        "shared_mean": float(np.mean([p["shared"] for p in per])),
        "saturated_mean": float(np.mean([p["saturated"] for p in per])),
        "shared_sat_mean": float(np.mean([p["shared_sat"] for p in per])),
        "shared_min": float(np.min([p["shared"] for p in per])),
        "shared_max": float(np.max([p["shared"] for p in per])),
        "seconds": round(time.time() - t0, 1),
        "per_pair": per,
    }
    print(json.dumps({k: v for k, v in out.items() if k != "per_pair"}))
    if args.json:
        with open(args.json, "w") as f:
            json.dump(out, f, indent=1)
    return out


if __name__ == "__main__":
    main()
