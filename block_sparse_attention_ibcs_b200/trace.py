"""Per-tile pipeline trace of the attention kernel (``ab_attn_debug`` with a trace buffer).

    python -m block_sparse_attention_ibcs_b200.trace [--workload wan14b] [--reps 3]

Runs select and plan on a synthetic workload, then the traced attention kernel, and prints
one JSON object: for each traced CTA (0, 1 and the one a third into the grid) the median
over its steady tiles (8 .. T-5) of every event's clock64 time after the tile's copy start,
the tile period, and the CTA's fill (copy start of tile 0 to its first QK and S) and drain
(its last PV to the CTA's end).  The event numbers are those ``include/abattn.h`` documents
for ``ab_attn_debug``.  The traced kernel is a separately compiled copy; its O equals the
untraced kernel's bit for bit, and its clock reads lengthen the tile period by a few
percent.
"""

import argparse
import json
import statistics

EVENTS = {
    0: "copy_start", 1: "copy_issued", 2: "sm_loaded", 3: "sm_exp_done", 4: "k_landed",
    5: "qk_issued", 6: "sm_pbuf", 7: "pv_issued", 8: "sm_start", 9: "sm_ready",
    10: "p_stored_w0", 11: "end", 12: "v_landed", 13: "p_stored_w1", 14: "p_stored_w2",
    15: "p_stored_w3",
}
SLOTS, EVENTS_PER_SLOT, TILES = 3, 16, 128


def summarize(trace, T):
    """Summary of a trace buffer (a flat sequence of 3*16*128 clock64 values, slot-major,
    then event, then tile) for T tiles per query block."""
    if T < 14:
        raise ValueError("the steady-state window needs at least 14 tiles per query block")
    whole = T <= TILES  # the block's last tile was traced too
    T = min(T, TILES)
    out = {}
    for slot in range(SLOTS):
        ev = [[int(trace[(slot * EVENTS_PER_SLOT + e) * TILES + t]) for t in range(TILES)]
              for e in range(EVENTS_PER_SLOT)]
        base = ev[0]
        steady = range(8, T - 5)
        rel = {}
        for e, name in EVENTS.items():
            if name == "end":
                continue
            rel[name] = statistics.median(ev[e][t] - base[t] for t in steady)
        rel["period"] = statistics.median(base[t + 1] - base[t] for t in steady)
        rel["fill_to_first_qk"] = ev[5][0] - base[0]
        rel["fill_to_first_s"] = ev[9][0] - base[0]
        if whole:
            rel["drain_last_pv_to_end"] = ev[11][0] - ev[7][T - 1]
            span = ev[11][0] - base[0]
            rel["cta_cycles"] = span
            rel["outside_steady_frac"] = round(1.0 - rel["period"] * T / span, 4) if span > 0 else None
        out[f"cta_slot{slot}"] = rel
    return out


def main():
    import torch

    import block_sparse_attention_ibcs_b200 as ab
    from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv

    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="wan14b", choices=sorted(WORKLOADS))
    ap.add_argument("--reps", type=int, default=3, help="traced calls; the last one is summarized")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    Q, K, V = make_qkv(w, device="cuda")
    p = ab.params(w.B, w.H, w.N, w.d, w.kv_block)
    rows = w.B * w.H * w.nQ
    S = torch.empty(w.B, w.H, w.nQ, w.nK, device="cuda")
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    idx = torch.empty(rows, w.s, dtype=torch.int32, device="cuda")
    lp = torch.empty(rows, w.s, device="cuda")
    ab.ab_select(p, Q, K, S, ws)
    ab.ab_plan(p, S, w.s, w.philox_seed, 0, idx, lp)
    del S, ws
    O = torch.empty_like(Q)
    tr = None
    for _ in range(max(1, args.reps)):
        tr = torch.zeros(SLOTS * EVENTS_PER_SLOT * TILES, dtype=torch.int64, device="cuda")
        ab.ab_attn_debug(p, Q, K, V, idx, lp, w.s, O, 0, 2_000_000_000, tr)
        st = ab.ab_get_status()
        if st != 0:
            raise RuntimeError(f"device status: {ab.ab_status_string(st)}")
    T = (w.s * w.kv_block + 127) // 128
    out = {"workload": w.name, "tiles_per_query_block": T, "unit": "SM clock cycles"}
    out.update(summarize(tr.cpu().tolist(), T))
    print(json.dumps(out))


if __name__ == "__main__":
    main()
