"""Benchmark of the AB-Attention hot path on B200 (one JSON line on rank 0).

One step = one pass of the whole hot path on the Wan2.1-14B-shaped layer
(B=1, H=40, N=75,600 = 21x45x80, d=128, KV block 4, s=2048 of 18,900 blocks kept):
  ab_select(Q, K) -> S, ab_plan(S) -> (idx, logpi), then 4 ab_attn calls reusing the
  plan, as the page reuses a plan for 4 denoising steps: the first on the Q/K/V the plan
  was selected on, the next three on perturbed copies (sigma 0.05, the drift of the
  following steps).
Inputs are synthetic (random-Fourier Q/K + noise, Gaussian V), generated on the
device before timing; every tensor is larger than L2, so no flush is needed.

Multi-GPU (torchrun), sharded by heads with no data-path collective (every (b, h) is
independent): by default a layer of H * N heads over N ranks, H heads each (weak scaling);
with --shard strong the configured layer's H heads split over the ranks (strong scaling).
Each rank calls the library on its own heads with head0 / heads_total set, so its S, plan
and O equal the matching rows of a one-GPU run over the whole layer.  The step time is the
max over ranks.

--impl reference times the CPU oracle (the only reference implementation: the pages
publish no code) on a bounded sample of the same workload, on rank 0.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/call and kept-block TFLOP/s (% bf16 peak) for ab_attn; select+plan GB/s (% HBM)"
UNIT = "TFLOP/s"  # kept-block attention FLOPs per second over the whole step


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    """Max of a host scalar over all ranks (NCCL on the GPU, gloo on the CPU)."""
    import torch

    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_heads(H, world, rank):
    """Head-parallel split of one layer: contiguous head range of this rank."""
    base, extra = divmod(H, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def rank_heads(w, world, rank, shard):
    """(head0, head1, heads_total) of this rank.  "weak": a layer of w.H * world heads, w.H
    per rank; "strong": the layer's w.H heads split over the ranks."""
    if shard == "strong":
        h0, h1 = shard_heads(w.H, world, rank)
        return h0, h1, w.H
    h0, h1 = shard_heads(w.H * world, world, rank)
    return h0, h1, w.H * world


def kept_flops(w, heads=None):
    """Kept-block attention FLOPs of one ab_attn call over `heads` heads (default w.H):
    4 * B * heads * N * (s * bk) * d."""
    return 4.0 * w.B * (w.H if heads is None else heads) * w.N * (w.s * w.kv_block) * w.d


def gathered_bytes(w, heads=None):
    """K and V bytes one ab_attn call gathers: every query block reads s*bk tokens of each."""
    return 2.0 * w.B * (w.H if heads is None else heads) * w.nQ * (w.s * w.kv_block) * w.d * 2


def attn_source_sha256():
    """Hash of the attention kernel's sources (the kernel and the helpers it inlines)."""
    h = hashlib.sha256()
    for f in ("attn.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "block_sparse_attention_ibcs_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


# DRAM bytes of one attention launch at the Wan2.1-14B shape from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum of the Wan2.1-1.3B-shaped launch, scaled by
# the number of heads: every head's K, V, Q and O cross DRAM once), valid only for the
# kernel source it was taken on; `roofline.traffic` is null for any other source.
ATTN_TRAFFIC = {"bytes_wan14b": 1.0385e9 * 40 / 12, "captured_heads": 12,
                "source_sha256": "9859efbd2b44054afd8d36c13896fbc5c2c29d6fb2033817e91b61716d6adebf"}


def attn_traffic(w, heads):
    t = ATTN_TRAFFIC
    if t["bytes_wan14b"] is None or t["source_sha256"] != attn_source_sha256():
        return None
    if (w.N, w.d, w.s, w.kv_block) != (75600, 128, 2048, 4):
        return None
    return round(t["bytes_wan14b"] * heads / 40.0)


def select_plan_bytes(w, heads=None):
    """Algorithmic HBM bytes of select+plan: |Q| + |K| (bf16) + 2|S| (fp32) + |idx| + |logpi|."""
    H = w.H if heads is None else heads
    qk = 2 * w.B * H * w.N * w.d * 2
    S = w.B * H * w.nQ * w.nK * 4
    plan = w.B * H * w.nQ * w.s * 8
    return qk + 2 * S + plan


def run_ours(args, world, rank, local):
    import torch

    import block_sparse_attention_ibcs_b200 as ab
    from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv, perturb

    w = WORKLOADS[args.workload]
    peaks = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    # this rank's heads of the (possibly larger) layer; inputs are drawn per global head
    h0, h1, Ht = rank_heads(w, world, rank, args.shard)
    Hr = h1 - h0
    Q, K, V = make_qkv(w, device=dev, heads=range(h0, h1))
    reuse = max(1, w.plan_reuse)
    # attention inputs of the plan's 4 steps: the refresh step's own Q/K/V, then drifted ones
    pert = [(Q, K, V)]
    for c in range(1, reuse):
        if w.perturb_sigma > 0:
            pert.append(tuple(perturb(x, w.perturb_sigma, 7000 + 10 * c + k + 100000 * rank)
                              for k, x in enumerate((Q, K, V))))
        else:
            pert.append((Q, K, V))
    p = ab.params(w.B, Hr, w.N, w.d, w.kv_block, w.clusters, w.kmeans_iters, head0=h0,
                  heads_total=Ht)
    rows = w.B * Hr * w.nQ
    S = torch.empty(w.B, Hr, w.nQ, w.nK, device=dev)
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device=dev)
    idx = torch.empty(rows, w.s, dtype=torch.int32, device=dev)
    lp = torch.empty(rows, w.s, device=dev)
    Os = [torch.empty_like(Q) for _ in range(reuse)]
    stream = torch.cuda.current_stream()

    ev = {}

    def E():
        return torch.cuda.Event(enable_timing=True)

    only_attn = args.only == "attn"
    run_select = args.only in ("all", "select")
    run_plan = args.only in ("all", "plan")
    run_attn = args.only in ("all", "attn")
    if args.only != "all":  # stage-only runs (kernel profiling): make the inputs once
        ab.ab_select(p, Q, K, S, ws)
        ab.ab_plan(p, S, w.s, w.philox_seed, 0, idx, lp)

    def step(i, record):
        if record:
            e0, e1, e2 = E(), E(), E()
            e0.record(stream)
        if run_select:
            ab.ab_select(p, Q, K, S, ws)
        if record:
            e1.record(stream)
        if run_plan:
            ab.ab_plan(p, S, w.s, w.philox_seed, i, idx, lp)
        if record:
            e2.record(stream)
        att = []
        for c in range(reuse if run_attn else 0):
            qa, ka, va = pert[c]
            if record:
                a0, a1 = E(), E()
                a0.record(stream)
            ab.ab_attn(p, qa, ka, va, idx, lp, w.s, Os[c])
            if record:
                a1.record(stream)
                att.append((a0, a1))
        if record:
            ev.setdefault("steps", []).append((e0, e1, e2, att))

    for i in range(args.warmup):
        step(i, False)
    st = ab.ab_get_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {ab.ab_status_string(st)}")

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0, t1 = E(), E()
        t0.record(stream)
        for i in range(args.steps):
            step(args.warmup + i, True)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    st = ab.ab_get_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {ab.ab_status_string(st)}")
    ms_total = t0.elapsed_time(t1)
    ms_total = max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    sel_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1, e2, _ in ev["steps"])
    plan_ms = statistics.mean(e1.elapsed_time(e2) for e0, e1, e2, _ in ev["steps"])
    attn_ms = (statistics.mean(a0.elapsed_time(a1) for *_, att in ev["steps"] for a0, a1 in att)
               if run_attn else float("nan"))
    F = kept_flops(w, Hr)  # one attention call of this rank
    F_all = kept_flops(w, Ht if args.shard == "strong" else w.H * world)  # all ranks
    value = reuse * F_all / (ms_step * 1e-3) / 1e12
    attn_tflops = F / (attn_ms * 1e-3) / 1e12
    sp_bytes = select_plan_bytes(w, Hr)
    sp_gbs = sp_bytes / ((sel_ms + plan_ms) * 1e-3) / 1e9

    # select + plan overlapped across head groups on two streams (ab_select_plan), timed
    # after the step loop on the same inputs
    sp_over_ms = None
    if args.only == "all":
        s2 = torch.cuda.Stream(device=dev)
        for i in range(2):
            ab.ab_select_plan(p, Q, K, S, ws, w.s, w.philox_seed, i, idx, lp, groups=2, stream2=s2)
        torch.cuda.synchronize()
        o0, o1 = E(), E()
        o0.record(stream)
        for i in range(3):  # two head groups: the least slow split measured (no split is faster)
            ab.ab_select_plan(p, Q, K, S, ws, w.s, w.philox_seed, i, idx, lp, groups=2, stream2=s2)
        o1.record(stream)
        torch.cuda.synchronize()
        sp_over_ms = max_over_ranks(o0.elapsed_time(o1) / 3, world)
        st = ab.ab_get_status()
        if st != 0:
            raise RuntimeError(f"device status after select+plan: {ab.ab_status_string(st)}")
    # select's exponential work at the special-function rate (16 per clock per SM)
    sm_hz = (clk.summary().get("sm_mhz") or 1800.0) * 1e6
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sel_exp = 2 * w.clusters * w.B * Hr * w.nQ * w.nK
    sel_sfu_ms = sel_exp / (16 * n_sms * sm_hz) * 1e3

    # end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e and args.only == "all":
        e2e = run_e2e(args, w, p, Q, K, pert, reuse, world, dev, F_all, Hr)

    peak_t = peaks["bf16_tflops"]  # burst: each attention call is timed on its own
    peak_sus = peaks["bf16_tflops_sustained"]
    heads_desc = (f"heads {h0}-{h1 - 1} of {Ht} on rank {rank}" if world > 1 else f"H={w.H}")
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "strong" if args.shard == "strong" else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (random-Fourier Q/K + noise, Gaussian V; seeded)",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} ({'x'.join(map(str, w.latent))}) "
                               f"d={w.d} kv_block={w.kv_block} q_block=128 clusters={w.clusters} "
                               f"s={w.s}/{w.nK} plan_reuse={reuse}",
                   "global_batch": w.B, "seq_len": w.N,
                   "parallelism": (f"head-sharded x{world} ({'strong' if args.shard == 'strong' else 'weak'}: "
                                   f"{Ht} heads, {heads_desc})" if world > 1 else "1 GPU"),
                   "l2": "inputs larger than L2 (Q/K/V 774 MB each), no flush"},
        "ms_per_attn_call": round(attn_ms, 3),
        "attn_tflops": round(attn_tflops, 2),
        "attn_frac_of_bf16_peak": round(attn_tflops / peak_t, 4),
        "attn_frac_of_bf16_sustained_peak": round(attn_tflops / peak_sus, 4),
        "select_ms": round(sel_ms, 3), "plan_ms": round(plan_ms, 3),
        "select_plan_gbs": round(sp_gbs, 1),
        "select_plan_frac_of_hbm": round(sp_gbs / peaks["hbm_gbs"], 4),
        "select_sfu_bound_ms": round(sel_sfu_ms, 3),
        "select_sfu_frac": round(sel_sfu_ms / sel_ms, 4) if run_select else None,
        "select_plan_overlapped_ms": None if sp_over_ms is None else round(sp_over_ms, 3),
        "select_plan_overlapped_frac_of_hbm": (None if sp_over_ms is None else
                                               round(sp_bytes / (sp_over_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)),
        "roofline": {"bound": "tensor", "kernel": "attn_kernel<128,false>",
                     "achieved": round(attn_tflops, 2), "peak": peak_t, "unit": "TFLOP/s",
                     "frac": round(attn_tflops / peak_t, 4),
                     "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                     "frac_of_sustained": round(attn_tflops / peak_sus, 4),
                     "sustained_peak": peak_sus,
                     "traffic": attn_traffic(w, Hr),
                     "traffic_source_sha256": attn_source_sha256()[:16],
                     "l2_gather_gbs": round(gathered_bytes(w, Hr) / (attn_ms * 1e-3) / 1e9, 1)},
        "gpu_launches": args.steps * (4 * run_select + run_plan + 2 * reuse * run_attn),  # attention: plan check + attention
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, seconds=args.cpu_seconds)
    return out


def run_e2e(args, w, p, Q, K, pert, reuse, world, dev, F_all, Hr):
    """Same step through the public API with host inputs: H2D of every input, D2H of every O.
    The selector reads the first attention call's Q and K (the refresh step's own), so each
    step copies the 4 calls' Q/K/V once."""
    import torch

    import block_sparse_attention_ibcs_b200 as ab

    hostP = [tuple(x.cpu().pin_memory() for x in t) for t in pert]
    hostO = [torch.empty(Q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(reuse)]
    dP = [tuple(torch.empty_like(Q) for _ in range(3)) for _ in range(reuse)]
    rows = w.B * Hr * w.nQ
    S = torch.empty(w.B, Hr, w.nQ, w.nK, device=dev)
    ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device=dev)
    idx = torch.empty(rows, w.s, dtype=torch.int32, device=dev)
    lp = torch.empty(rows, w.s, device=dev)
    dO = [torch.empty_like(Q) for _ in range(reuse)]
    h2d = 3 * reuse * Q.numel() * 2
    d2h = reuse * Q.numel() * 2

    # Three streams: host->device copies (cs), compute (the current stream), device->host
    # copies (ds).  The copy of attention call c's inputs overlaps the calls before it, and
    # each output's copy back overlaps the calls after it; events keep every buffer from
    # being overwritten before its previous reader is done.
    stream = torch.cuda.current_stream()
    cs = torch.cuda.Stream(device=dev)
    ds = torch.cuda.Stream(device=dev)
    prev = {"attn": [None] * reuse, "d2h": [None] * reuse}

    def ev_on(st):
        e = torch.cuda.Event()
        e.record(st)
        return e

    def step(i):
        with torch.cuda.stream(cs):
            ready = []
            for c in range(reuse):
                # call c's buffers are free once the previous step's call c (and, for c = 0,
                # the selector before it on the same stream) has read them
                if prev["attn"][c] is not None:
                    cs.wait_event(prev["attn"][c])
                for dst, src in zip(dP[c], hostP[c]):
                    dst.copy_(src, non_blocking=True)
                ready.append(ev_on(cs))
        stream.wait_event(ready[0])
        ab.ab_select(p, dP[0][0], dP[0][1], S, ws, stream)
        ab.ab_plan(p, S, w.s, w.philox_seed, i, idx, lp, stream)
        for c in range(reuse):
            stream.wait_event(ready[c])
            if prev["d2h"][c] is not None:
                stream.wait_event(prev["d2h"][c])
            ab.ab_attn(p, dP[c][0], dP[c][1], dP[c][2], idx, lp, w.s, dO[c], stream)
            prev["attn"][c] = ev_on(stream)
            with torch.cuda.stream(ds):
                ds.wait_event(prev["attn"][c])
                hostO[c].copy_(dO[c], non_blocking=True)
                prev["d2h"][c] = ev_on(ds)

    for i in range(2):
        step(i)
    steps = max(1, args.steps)
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    cs.wait_stream(stream)  # nothing of the timed steps starts before t0
    ds.wait_stream(stream)
    for i in range(steps):
        step(100 + i)
    stream.wait_stream(cs)  # ... and t1 follows every copy of them
    stream.wait_stream(ds)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world)
    value = reuse * F_all / (ms * 1e-3) / 1e12
    return {"value": round(value, 3), "unit": UNIT, "ms_per_step": round(ms, 2), "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def oracle_threads():
    """Threads the oracle's numpy work runs on in one process: the BLAS thread pool
    (threadpoolctl), else torch's intra-op thread count."""
    try:
        import threadpoolctl

        n = [i.get("num_threads", 0) for i in threadpoolctl.threadpool_info()
             if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    import torch

    return torch.get_num_threads()


# ---- the oracle on all host cores: one worker process per core, one BLAS thread each.
# Workers start with "spawn" (a process forked after CUDA was initialised can hang) and
# each draws head 0 of the workload and pools its keys once, before the timed region.

_OB = {}


def _oracle_worker_init(name):
    import threadpoolctl

    from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv
    from oracle import abattn_oracle as O

    threadpoolctl.threadpool_limits(1)
    w = WORKLOADS[name]
    Q, K, V = make_qkv(w, device="cpu", heads=[0])
    q, k, v = (t[0, 0].double().numpy() for t in (Q, K, V))
    t0 = time.perf_counter()
    Kp = O.pool_keys(k, w.kv_block)
    _OB.update(w=w, q=q, k=k, v=v, Kp=Kp, pool_s=time.perf_counter() - t0)


def _oracle_worker_ping(_):
    time.sleep(0.2)
    return _OB["pool_s"]


def _oracle_query_block(i):
    """Select + plan + attention of query block i of head 0; returns its valid rows."""
    from oracle import abattn_oracle as O

    w, q, k, v, Kp = _OB["w"], _OB["q"], _OB["k"], _OB["v"], _OB["Kp"]
    Qb = q[i * 128: min(w.N, (i + 1) * 128)]
    cent, wt, _, _ = O.kmeans_block(Qb, w.clusters, w.kmeans_iters)
    S = O.block_scores(cent, wt, Kp).astype(np.float32)
    idx, lp, _ = O.plan_row(S, w.s, w.philox_seed, 0, i)
    O.attn_block(Qb, k, v, idx, lp, w.kv_block)
    return Qb.shape[0]


class OraclePool:
    """The oracle as it stands, parallel over query blocks on the host's cores."""

    def __init__(self, w, procs=None):
        import multiprocessing as mp

        self.w = w
        if procs is None:  # the cores this process may run on (at most 64 workers)
            try:
                procs = len(os.sched_getaffinity(0))
            except AttributeError:
                procs = os.cpu_count() or 1
            procs = max(1, min(64, procs))
        self.procs = procs
        self.pool = mp.get_context("spawn").Pool(self.procs, _oracle_worker_init, (w.name,))
        # every worker has drawn its inputs and pooled the keys before anything is timed
        pings = self.pool.map(_oracle_worker_ping, range(2 * self.procs), chunksize=1)
        self.pool_s = max(pings)
        self.order = [int(i) for i in np.random.default_rng(0).permutation(w.nQ)]
        self.next = 0

    def run(self, seconds):
        """Query blocks in a fixed order until about `seconds` of wall time have passed;
        returns (kept-block FLOP/s, description).  The head's key pooling, done once per
        worker, is charged in proportion to the query blocks processed."""
        w = self.w
        t0 = time.perf_counter()
        rows = done = 0
        while time.perf_counter() - t0 < seconds:
            batch = [self.order[(self.next + k) % w.nQ] for k in range(self.procs)]
            self.next += self.procs
            for r in self.pool.map(_oracle_query_block, batch, chunksize=1):
                rows += r
                done += 1
        dt = time.perf_counter() - t0 + self.pool_s * done / w.nQ
        flops = 4.0 * rows * (w.s * w.kv_block) * w.d
        sample = (f"head 0, {done} query blocks (k-means, scores, plan, attention per block; the "
                  f"head's key pooling charged pro rata), {self.procs} processes x 1 BLAS thread, "
                  f"{dt:.1f} s")
        return flops / dt, sample, 1e3 * dt * self.procs / done

    def close(self):
        self.pool.terminate()
        self.pool.join()


def cpu_baseline(w, seconds=15.0):
    """The oracle as it stands on all host cores (one process per core) for a bounded
    sample of query blocks of head 0, in the metric's unit (kept-block FLOP/s)."""
    pool = OraclePool(w)
    try:
        v, sample, ms_qb = pool.run(seconds)
    finally:
        pool.close()
    return {"value": round(v / 1e12, 6), "unit": UNIT, "cores": pool.procs, "kind": "oracle",
            "sample": sample, "ms_per_query_block_per_core": round(ms_qb, 1)}


def run_sweep(args):
    """Granularity sweep at the Wan2.1-1.3B shape (not a bench line; prints one JSON line).

    For KV block 4, 16, 64, 128 at a fixed budget of 8192 kept tokens per query block:
    packed tiles per query block (ceil(s*bk/128) = 64 in every case) against one tile
    per selected block (s), and select/plan/attention times.  Also times s = all blocks
    through the packed kernel against the same kernel's dense path.  (The error of each
    case against fp64 dense attention is measured by `tests/ablation_report.py --sweep`,
    which uses the oracle.)
    """
    import torch

    import block_sparse_attention_ibcs_b200 as ab
    from block_sparse_attention_ibcs_b200.inputs import WORKLOADS, make_qkv

    torch.cuda.set_device(0)
    base = WORKLOADS["sweep_bk4"]
    Q, K, V = make_qkv(base, device="cuda")
    stream = torch.cuda.current_stream()

    def timed(fn, reps=3):
        fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    out = {"workload": "Wan2.1-1.3B shape: B=1 H=12 N=75600 d=128, 8192 kept tokens per query block",
           "cases": []}
    for bk in (4, 16, 64, 128):
        w = WORKLOADS[f"sweep_bk{bk}"]
        p = ab.params(w.B, w.H, w.N, w.d, bk)
        R = w.B * w.H * w.nQ
        S = torch.empty(w.B, w.H, w.nQ, w.nK, device="cuda")
        ws = torch.empty(ab.ab_workspace_bytes(p), dtype=torch.uint8, device="cuda")
        idx = torch.empty(R, w.s, dtype=torch.int32, device="cuda")
        lp = torch.empty(R, w.s, device="cuda")
        Od = torch.empty_like(Q)
        t_sel = timed(lambda: ab.ab_select(p, Q, K, S, ws))
        t_plan = timed(lambda: ab.ab_plan(p, S, w.s, w.philox_seed, 0, idx, lp))
        t_attn = timed(lambda: ab.ab_attn(p, Q, K, V, idx, lp, w.s, Od))
        assert ab.ab_get_status() == 0
        out["cases"].append({"kv_block": bk, "s": w.s, "nK": w.nK,
                             "tiles_per_query_block_packed": -(-w.s * bk // 128),
                             "tiles_per_query_block_one_per_block": w.s,
                             "select_ms": round(t_sel, 3), "plan_ms": round(t_plan, 3),
                             "attn_ms": round(t_attn, 3),
                             "attn_tflops": round(kept_flops(w) / (t_attn * 1e-3) / 1e12, 1)})
    # s = all blocks through the packed kernel vs the dense path (bk = 128: 591 blocks)
    w = WORKLOADS["sweep_bk128"]
    p = ab.params(w.B, w.H, w.N, w.d, 128)
    R = w.B * w.H * w.nQ
    idx = torch.arange(w.nK, dtype=torch.int32, device="cuda").repeat(R, 1).contiguous()
    lp = torch.zeros(R, w.nK, device="cuda")
    O1, O2 = torch.empty_like(Q), torch.empty_like(Q)
    t_pk = timed(lambda: ab.ab_attn(p, Q, K, V, idx, lp, w.nK, O1), reps=2)
    t_dn = timed(lambda: ab.ab_attn_dense(p, Q, K, V, O2), reps=2)
    dense_flops = 4.0 * w.B * w.H * w.N * w.N * w.d
    out["all_blocks"] = {"packed_ms": round(t_pk, 3), "dense_path_ms": round(t_dn, 3),
                         "dense_tflops": round(dense_flops / (t_dn * 1e-3) / 1e12, 1),
                         "bitwise_equal": bool(torch.equal(O1, O2))}
    print(json_line(out), flush=True)


def json_line(obj):
    """The JSON line with every non-finite number as null (a stage-only run leaves the
    stages it did not time as NaN), so that strict parsers accept it."""
    def clean(x):
        if isinstance(x, float) and not math.isfinite(x):
            return None
        if isinstance(x, dict):
            return {k: clean(v) for k, v in x.items()}
        if isinstance(x, (list, tuple)):
            return [clean(v) for v in x]
        return x
    return json.dumps(clean(obj), allow_nan=False)


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle (the pages publish no implementation)."""
    if rank != 0:
        return None
    from block_sparse_attention_ibcs_b200.inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    per = getattr(args, "ref_seconds", None) or max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    vals = []
    pool = OraclePool(w)
    try:
        for i in range(args.warmup + args.steps):
            v, sample, _ = pool.run(per)
            if i >= args.warmup:
                vals.append({"value": v / 1e12, "sample": sample})
    finally:
        pool.close()
    value = statistics.mean(c["value"] for c in vals)
    ms_step = 1e3 * 4.0 * w.B * w.H * w.N * (w.s * w.kv_block) * w.d * max(1, w.plan_reuse) / (value * 1e12)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": f"{w.name} (bounded sample per step, extrapolated)",
                       "global_batch": w.B, "seq_len": w.N, "parallelism": "cpu"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": pool.procs,
                             "kind": "oracle", "sample": vals[0]["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="wan14b")
    ap.add_argument("--only", default="all", choices=["all", "attn", "select", "plan"],
                    help="time one stage only (kernel profiling); the step is then that stage")
    ap.add_argument("--sweep", action="store_true",
                    help="granularity sweep (KV block 4..128) at the Wan2.1-1.3B shape")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="reference arm: seconds of oracle work per step (default: 60 s over all steps)")
    ap.add_argument("--shard", default="weak", choices=["weak", "strong"],
                    help="N>1: a layer of H*N heads, H per rank (weak), or the layer's H heads "
                         "split over the ranks (strong)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json_line(out), flush=True)
        return
    world, rank, local = dist_setup(args)
    out = run_ours(args, world, rank, local)
    if rank == 0:
        print(json_line(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
