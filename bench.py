#!/usr/bin/env python
"""Benchmark of one InstaGen attention call (cluster Q and K, permute/gather,
select + group-shared sample, sparse attention) on B200.

Metric: ms per attention call (lower is better), plus effective TFLOP/s on the
attended FLOPs (sum over heads and query groups of 4 * n_i * (exact_i + m) * d)
as a fraction of the measured bf16 tensor-core peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the CPU oracle, bounded sample)

Multi-GPU: the call does not shard across GPUs (one call per GPU); N ranks run
N independent calls (replicas, one layer each), no collective on the data
path; value = aggregate ms per call = max-over-ranks time / (K * N).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="instagen", choices=["instagen", "reference"])
    ap.add_argument("--workload", default="wan2.1-14b_720p")
    ap.add_argument("--exact", type=float, default=None, help="override the exact share")
    ap.add_argument("--sample", type=float, default=None, help="override the sampled share")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the head count (same per-head shape; for profiling captures)")
    ap.add_argument("--selection", default="centroid", choices=["centroid", "pq_vote"],
                    help="exact-set ranking: centroid scores (default) or product-quantised per-query votes")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-sweeps", action="store_true",
                    help="skip the untimed budget points added to the line (density ends, sample sweep)")
    ap.add_argument("--sweep", action="store_true",
                    help="budget sweep (error vs dense SDPA and ms per call per budget, one JSON line "
                         "each) and a warm-started call; not part of the default run")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, source="fallback")


def attention_traffic_per_unit():
    """DRAM bytes per attended key-row (from the committed ncu summary) if it was
    captured on the current attention kernel source, else None."""
    path = os.path.join(ROOT, "profiles", "attention_traffic.json")
    src = os.path.join(ROOT, "block_sparse_attention_head_b200", "csrc", "attention.cu")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    if d.get("attention_cu_sha256") != h:
        return None
    return d


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"instagen_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={SMI_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx, "samples": len(mhz),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------- CPU oracle
class OracleSample:
    """The CPU oracle on a bounded sample of the workload (one head).

    The head's inputs are drawn exactly as the GPU arm draws them (the same
    seeded generator on the GPU when one is present, so both arms see the same
    tensors), then copied to the host.  Set-up (untimed): one oracle k-means
    iteration, whose centroids and lists feed the timed stages.  One timed
    step: k-means assign + update of 4096 sampled tokens against the Q and K
    centroids (x N/4096 tokens, x iters), select/sample of the head's query
    groups, and attention for 32 query rows (x N/32); extrapolated x B*H heads.
    """

    def __init__(self, w, exact, sample, seed=0, layer=0):
        import numpy as np
        import oracle
        from block_sparse_attention_head_b200 import workloads
        import torch
        oracle.build()
        self.np, self.oracle, self.w = np, oracle, w
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        self.input_device = dev
        Q, K, V = workloads.make_inputs(w, heads=[0], layer=layer, device=dev)
        self.Q, self.K, self.V = (t[0, 0].float().cpu().numpy() for t in (Q, K, V))
        self.scale = 1.0 / math.sqrt(w.d)
        self.cq, self.qa, _ = oracle.kmeans(self.Q, w.Cq, 1)
        self.ck, self.ka, _ = oracle.kmeans(self.K, w.Ck, 1)
        self.kp, self.ko = oracle.permutation(self.ka, w.Ck)
        self.E, self.m = oracle.budget(exact, w.N), oracle.budget(sample, w.N)
        self.seed = seed
        self.rng = np.random.default_rng(0)
        self.n_tok, self.n_rows = min(4096, w.N), min(32, w.N)

    def step(self):
        o, w, np = self.oracle, self.w, self.np
        tok = self.rng.choice(w.N, self.n_tok, replace=False)
        t0 = time.perf_counter()
        for X, cent in ((self.Q, self.cq), (self.K, self.ck)):
            xs = np.ascontiguousarray(X[tok])
            a, _ = o.kmeans_assign(xs, cent)
            o.kmeans_update(xs, a, cent)
        t_km = time.perf_counter() - t0
        t1 = time.perf_counter()
        ex, cnt, sp, sb = o.select_sample(self.cq, self.ck, self.ko, self.scale, self.E, self.m, seed=self.seed)
        t_sel = time.perf_counter() - t1
        rows = self.rng.choice(w.N, self.n_rows, replace=False)
        t2 = time.perf_counter()
        o.attention_rows(self.Q, self.K, self.V, self.scale, self.qa, self.kp, self.ko, ex, cnt, sp, sb, rows)
        t_att = time.perf_counter() - t2
        per_head = t_km * (w.N / self.n_tok) * w.iters + t_sel + t_att * (w.N / self.n_rows)
        return per_head * w.B * w.H * 1e3

    def describe(self):
        w = self.w
        return (f"head 0 of {w.name} (inputs drawn on {self.input_device} as the GPU arm draws them): k-means "
                f"assign+update of {self.n_tok} tokens for Q and K (x{w.N / self.n_tok:.1f} tokens, x{w.iters} "
                f"iterations), select/sample of the head, attention on {self.n_rows} query rows "
                f"(x{w.N / self.n_rows:.0f}); extrapolated x{w.B * w.H} heads")

    def fields(self):
        """Machine-readable description of the extrapolation."""
        w = self.w
        return {"extrapolated": True, "heads_timed": 1, "heads_total": w.B * w.H,
                "kmeans_tokens_timed": self.n_tok, "attention_rows_timed": self.n_rows, "tokens": w.N,
                "input_device": self.input_device}


def reference_arm(args, w, exact, sample):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    t0 = time.perf_counter()
    orc = OracleSample(w, exact, sample)
    for _ in range(args.warmup):
        orc.step()
    vals = [orc.step() for _ in range(args.steps)]
    ms = statistics.median(vals)
    line = {
        "impl": "reference", "metric": "ms per InstaGen attention call", "value": round(ms, 1),
        "unit": "ms/call", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, exact, sample),
        "cpu_baseline": {"kind": "oracle", "cores": orc.oracle.num_threads(), "sample": orc.describe(),
                         "value": round(ms, 1), "unit": "ms/call", **orc.fields()},
        "e2e": {"value": round(ms, 1), "unit": "ms/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(time.perf_counter() - t0, 1),
    }
    print(json.dumps(line))
    return 0


def max_over_ranks(vals, dist=None, device="cpu"):
    """Element-wise maximum over all ranks of a list of per-rank floats (the
    list itself with one rank); every rank gets the same result."""
    if dist is None:
        return [float(v) for v in vals]
    import torch
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_time(t_total_ms, e2e_ms_per_call, steps, world, dist=None, device="cpu"):
    """Whole-job timing of `world` replicas that each ran `steps` calls: the
    slowest rank's device time sets the job's time, so
    ms_call = max(t_total) / steps is one rank's time per call and the
    aggregate ms per call is ms_call / world (world calls per step); the end
    to end time per call is aggregated the same way.  Returns
    (ms_call, aggregate ms/call, aggregate e2e ms/call)."""
    t_max, e2e_max = max_over_ranks([t_total_ms, e2e_ms_per_call], dist, device)
    ms_call = t_max / steps
    return ms_call, ms_call / world, e2e_max / world


def budget_point(ig, Q, K, V, w, exact, sample, D, dn, *, seed, layer, reps=3, ws=None, **sel):
    """ms per instagen_forward call (CUDA events, one warm-up, median of
    `reps`) and the relative L2 error of its output against the dense output
    D (||D|| = dn) for one (exact, sample) budget on the given inputs; also
    the attended density of the call.  ``sel``: selection keywords of
    make_params (e.g. selection="top_p", top_p=0.9, key_floor=0.1)."""
    import torch
    p = ig.make_params(w.B, w.H, w.N, w.d, w.Cq, w.Ck, iters=w.iters, exact_frac=exact, sample_frac=sample,
                       seed=seed, layer=layer, **sel)
    if ws is None or ws.numel() < ig.workspace_size(p):
        ws = torch.empty(ig.workspace_size(p), dtype=torch.uint8, device=Q.device)
    O = torch.empty_like(Q)
    ig.forward(Q, K, V, p, workspace=ws, out=O)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        ig.forward(Q, K, V, p, workspace=ws, out=O)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ig.device_status()
    err = float((O.float() - D).pow(2).sum().sqrt()) / dn
    it = ig.forward_intermediates(ws, p)
    cnt = it["counts"].long()
    qoff = it["q_offsets"].long()
    pairs = float(((qoff[..., 1:] - qoff[..., :-1]) * (cnt[..., 1] + cnt[..., 2])).sum())
    out = {"exact_frac": exact, "sample_frac": sample, "ms_per_call": round(statistics.median(ts), 3),
           "rel_l2_vs_dense": round(err, 4), "density": round(pairs / (w.B * w.H * w.N * w.N), 4)}
    if sel:
        out.update({k: v for k, v in sel.items()})
        out.pop("exact_frac")
        out.pop("sample_frac")
    return out


def top_p_comparator(ig, Q, K, V, w, D, dn, rank):
    """The SVG2-style top-p selection (no sample; key floor 0.1) at p = 0.5,
    0.75, 0.9, 0.95, each beside the importance-sampled call at the same
    attended density (exact and sampled shares each half of that density):
    ms per call and error against dense attention."""
    rows = []
    for tp in (0.5, 0.75, 0.9, 0.95):
        a = budget_point(ig, Q, K, V, w, 0.0, 0.0, D, dn, seed=1000 + rank, layer=rank, selection="top_p",
                         top_p=tp, key_floor=0.1)
        half = round(a["density"] / 2, 4)
        b = budget_point(ig, Q, K, V, w, half, half, D, dn, seed=1000 + rank, layer=rank)
        rows.append({"top_p": a, "importance_at_matched_density": b})
    return rows


def stack_sample_sweep(ig, dev, args):
    """The 40-layer Wan2.1-14B stack's sample-budget sweep (exact 8%, sampled
    2 to 32%) on one full 40-head layer of it (layer 0, its own seeded
    mixture): ms per call and error against dense attention per budget, plus
    the exact-only call at 8%."""
    import torch
    import torch.nn.functional as F
    from block_sparse_attention_head_b200 import workloads
    ws_ = workloads.WAN14B_STACK
    Q, K, V = workloads.make_inputs(ws_, layer=0, device=dev)
    D = F.scaled_dot_product_attention(Q, K, V, scale=ws_.softmax_scale).float()
    dn = float(D.pow(2).sum().sqrt())
    pts = [budget_point(ig, Q, K, V, ws_, ex, sa, D, dn, seed=11, layer=0) for ex, sa in ws_.sweep]
    pts.append(budget_point(ig, Q, K, V, ws_, ws_.exact_frac, 0.0, D, dn, seed=11, layer=0))
    del Q, K, V, D
    torch.cuda.empty_cache()
    return {"workload": ws_.name, "layers_run": 1, "layer": 0, "heads": ws_.B * ws_.H,
            "note": "one full 40-head layer of the 40-layer stack; the other layers share its shape and recipe",
            "points": pts}


def workload_config(w, exact, sample, selection="centroid"):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "Cq": w.Cq, "Ck": w.Ck,
            "kmeans_iters": w.iters, "exact_frac": exact, "sample_frac": sample, "sampling": "importance",
            "selection": selection,
            "inputs": "clustered Gaussian mixture (seeded), bf16",
            "l2": "inputs (Q,K,V %.1f GB per call) larger than L2" % (3 * w.B * w.H * w.N * w.d * 2 / 1e9)}


# ------------------------------------------------------------------ GPU arm
def main():
    args = parse_args()
    from block_sparse_attention_head_b200 import workloads
    w = workloads.WORKLOADS[args.workload]
    if args.heads is not None:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads)
    exact = w.exact_frac if args.exact is None else args.exact
    sample = w.sample_frac if args.sample is None else args.sample
    if args.impl == "reference":
        return reference_arm(args, w, exact, sample)
    if args.sweep:
        return sweep_mode(args, w)

    import torch
    import block_sparse_attention_head_b200 as ig
    from block_sparse_attention_head_b200 import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    build.build()
    ig.lib()

    peaks = load_peaks()
    dev = torch.device("cuda", local)
    Q, K, V = workloads.make_inputs(w, layer=rank, device=dev)
    p = ig.make_params(w.B, w.H, w.N, w.d, w.Cq, w.Ck, iters=w.iters, exact_frac=exact, sample_frac=sample,
                       seed=1000 + rank, layer=rank, selection=args.selection)
    pq = args.selection == "pq_vote"
    ws = torch.empty(ig.workspace_size(p), dtype=torch.uint8, device=dev)
    O = torch.empty_like(Q)
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    # ---------------- headline: instagen_forward, inputs resident in HBM
    for _ in range(args.warmup):
        ig.forward(Q, K, V, p, workspace=ws, out=O)
    ig.device_status()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            ig.forward(Q, K, V, p, workspace=ws, out=O)
        ev1.record(stream)
        barrier()
    ig.device_status()
    t_fwd = ev0.elapsed_time(ev1)
    clocks = clk.summary()

    # ---------------- stage breakdown: the same calls, staged, with events
    inter = ig.forward_intermediates(ws, p)
    stages = ["cluster_q", "cluster_k", "gather_kv"] + (["pq_votes"] if pq else []) + ["select_sample", "attention"]
    acc = {s: 0.0 for s in stages}
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
    barrier()
    # one untimed pass first: the staged calls allocate their outputs, and a
    # first allocation that blocks the host would sit inside a stage's events
    for it in range(args.steps + 1):
        timed = it > 0
        evs[0].record(stream)
        cq, qa, qp, qo = ig.cluster(Q, w.Cq, w.iters, p)
        evs[1].record(stream)
        ck, ka, kp, ko = ig.cluster(K, w.Ck, w.iters, p)
        evs[2].record(stream)
        Kp, Vp = ig.gather(K, kp, p), ig.gather(V, kp, p, to_f16=True)
        evs[3].record(stream)
        votes = None
        if pq:
            votes = ig.pq_votes(Q, cq, ck, qp, qo, ko, p)
            evs[4].record(stream)
        eg, cnt, sp, sb = ig.select_sample(cq, ck, ko, p, votes=votes)
        evs[len(stages) - 1].record(stream)
        ig.attention(Q, Kp, Vp, qp, qo, ko, eg, cnt, sp, sb, p, out=O)
        evs[len(stages)].record(stream)
        torch.cuda.synchronize()
        for i, s in enumerate(stages):
            acc[s] += evs[i].elapsed_time(evs[i + 1]) if timed else 0.0
        del cq, qa, qp, qo, ck, ka, kp, ko, Kp, Vp, eg, cnt, sp, sb
    ig.device_status()
    stage_ms = {s: acc[s] / args.steps for s in stages}

    # ---------------- algorithmic work (from the call's own lists)
    counts = inter["counts"].long().cpu()
    qoff = inter["q_offsets"].long().cpu()
    n_i = (qoff[..., 1:] - qoff[..., :-1])
    keys_i = counts[..., 1] + counts[..., 2]
    attended_flops = float((4 * n_i * keys_i * w.d).sum())
    attended_rows = float((n_i * keys_i).sum())          # (query, key) pairs
    key_tile_loads = float((((n_i + 127) // 128) * keys_i).sum())  # K/V rows streamed per query tile
    density = attended_rows / (w.B * w.H * w.N * w.N)
    t_att = stage_ms["attention"]
    achieved = attended_flops / (t_att * 1e-3) / 1e12
    # HBM-side stages: algorithmic bytes
    BH, N, d = w.B * w.H, w.N, w.d
    m = ig.sample_budget(p)
    # k-means: one read of the tokens and one int32 assignment per token per
    # iteration (the method's algorithmic traffic; the update's second pass
    # over the tokens is not counted)
    bytes_cluster = lambda C: w.iters * (BH * N * d * 2 + BH * N * 4)
    hbm = {
        "cluster_q": bytes_cluster(w.Cq), "cluster_k": bytes_cluster(w.Ck),
        "gather_kv": 2 * 2 * BH * N * d * 2 + BH * N * 4,
        "select_sample": BH * w.Cq * (m * 8 + w.Ck * 4) + BH * (w.Cq + w.Ck) * d * 4,
    }
    stage_report = {}
    for s in stages:
        e = {"ms": round(stage_ms[s], 3)}
        if s in hbm:
            gbs = hbm[s] / (stage_ms[s] * 1e-3) / 1e9
            e.update(algorithmic_bytes=int(hbm[s]), gbs=round(gbs, 1), hbm_frac=round(gbs / peaks["hbm"], 3),
                     hbm_peak_gbs=peaks["hbm"])
        stage_report[s] = e
    kmeans_flops = 2 * BH * N * (w.Cq + w.Ck) * d * 2 * w.iters     # hi+lo operand: K = 2d
    stage_report["cluster_q"]["tensor_tflops"] = round(
        2 * BH * N * w.Cq * d * 2 * w.iters / (stage_ms["cluster_q"] * 1e-3) / 1e12, 1)
    stage_report["cluster_k"]["tensor_tflops"] = round(
        2 * BH * N * w.Ck * d * 2 * w.iters / (stage_ms["cluster_k"] * 1e-3) / 1e12, 1)

    traffic = None
    tr = attention_traffic_per_unit()
    if tr is not None and tr.get("workload") == w.name and abs(tr.get("exact_frac", -1) - exact) < 1e-9 \
            and abs(tr.get("sample_frac", -1) - sample) < 1e-9:
        traffic = tr["dram_bytes_per_launch"]

    # ---------------- dense comparator (torch SDPA) and error vs dense
    extra = {}
    if not args.no_dense:
        import torch.nn.functional as F
        for _ in range(2):
            D = F.scaled_dot_product_attention(Q, K, V, scale=p.softmax_scale)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            D = F.scaled_dot_product_attention(Q, K, V, scale=p.softmax_scale)
        e1.record(stream)
        torch.cuda.synchronize()
        extra["dense_sdpa_ms"] = round(e0.elapsed_time(e1) / 3, 3)
        ig.forward(Q, K, V, p, workspace=ws, out=O)
        num = (O.float() - D.float()).pow(2).sum().sqrt()
        den = D.float().pow(2).sum().sqrt()
        extra["rel_l2_vs_dense"] = round(float(num / den), 4)
        if not args.no_sweeps and not pq:
            # density ends of the budget range on the same inputs (untimed
            # for the headline value; each point timed on its own)
            Df = D.float()
            dn = float(Df.pow(2).sum().sqrt())
            extra["density_sweep"] = [budget_point(ig, Q, K, V, w, ex, sa, Df, dn, seed=1000 + rank, layer=rank,
                                                   ws=ws)
                                      for ex, sa in ((0.04, 0.04), (0.32, 0.32))]
            extra["top_p_comparator"] = top_p_comparator(ig, Q, K, V, w, Df, dn, rank)
            del Df
        del D

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        # instagen_forward_host: pinned host Q/K/V in, host O out; head chunks
        # are copied in, computed and copied out as a pipeline
        hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
        hO = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
        del ws  # the device workspace of the device-buffer call is not needed here
        hws = torch.empty(ig.forward_host_workspace_size(p), dtype=torch.uint8, device=dev)

        def e2e_step():
            ig.forward_host(hQ, hK, hV, p, out=hO, workspace=hws)

        for _ in range(2):
            e2e_step()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        ksteps = max(1, min(args.steps, 5))
        for _ in range(ksteps):
            e2e_step()
        a1.record(stream)
        barrier()
        t_e2e = a0.elapsed_time(a1) / ksteps
        e2e = {"value": t_e2e, "unit": "ms/call", "h2d_bytes_per_step": 3 * Q.numel() * 2,
               "d2h_bytes_per_step": O.numel() * 2, "steps": ksteps}
        del hQ, hK, hV, hO, hws

    # ---------------- the stack's sample-budget sweep (untimed for the value)
    if not args.no_dense and not args.no_sweeps and not pq and args.heads is None and w.name == "wan2.1-14b_720p":
        extra["stack_sample_sweep"] = stack_sample_sweep(ig, dev, args)

    # ---------------- max over ranks
    ms_call, value, e2e_value = job_time(t_fwd, e2e["value"] if e2e else 0.0, args.steps, world, dist, dev)
    if e2e:
        e2e["value"] = e2e_value

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not pq:  # the sample runs the centroid ranking
        orc = OracleSample(w, exact, sample, layer=rank)
        orc.step()
        vals = [orc.step() for _ in range(3)]
        cpu = {"value": round(statistics.median(vals), 1), "unit": "ms/call", "cores": orc.oracle.num_threads(),
               "kind": "oracle", "sample": orc.describe() + "; median of 3 steps", **orc.fields()}

    launches_per_step = 2 * (1 + 3 * w.iters) + 1 + 1 + 1 + (2 if pq else 0)  # + codebooks, votes
    peak = peaks["bf16"]  # the burst figure: the kernel is timed per call, not in a seconds-long loop
    clk_frac = (clocks["sm_mhz"] / clocks["sm_max_mhz"]) if clocks.get("sm_mhz") and clocks.get("sm_max_mhz") else None
    line = {
        "metric": "ms per InstaGen attention call", "value": round(value, 3), "unit": "ms/call",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_call, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, exact, sample, args.selection),
        "effective_tflops": round(attended_flops / (ms_call * 1e-3) / 1e12, 1),
        "attended_flops": attended_flops, "density": round(density, 4),
        "roofline": {"kernel": "attention", "bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_kind": f"bf16 burst ({peaks['source']})",
                     "frac_clock_matched": (round(achieved / (peak * clk_frac), 4) if clk_frac else None),
                     "clock_matched_peak": (round(peak * clk_frac, 1) if clk_frac else None),
                     "frac_of_sustained": round(achieved / peaks["bf16_sust"], 4),
                     "traffic": traffic, "algorithmic_unit": "4*d FLOPs per attended (query,key) pair",
                     "flops_per_launch": attended_flops, "ms": round(t_att, 3)},
        "stages": stage_report,
        "e2e": ({"value": round(e2e["value"], 3), "unit": "ms/call", "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                 "d2h_bytes_per_step": e2e["d2h_bytes_per_step"]} if e2e else None),
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        **extra,
    }
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def sweep_mode(args, w):
    """Budget sweep on one GPU: for each (exact, sample) share, ms per call and
    the relative L2 error of O against dense attention (torch SDPA on the same
    bf16 inputs); exact-only calls at the same key share for comparison; and a
    call warm-started from the previous call's centroids with 2 k-means
    iterations instead of 10."""
    import torch
    import torch.nn.functional as F
    import block_sparse_attention_head_b200 as ig
    from block_sparse_attention_head_b200 import build, workloads
    build.build()
    ig.lib()
    dev = torch.device("cuda", 0)
    Q, K, V = workloads.make_inputs(w, device=dev)
    scale = 1.0 / math.sqrt(w.d)
    D = F.scaled_dot_product_attention(Q, K, V, scale=scale).float()
    dn = float(D.pow(2).sum().sqrt())

    def run(exact, sample, iters=w.iters, init=None):
        p = ig.make_params(w.B, w.H, w.N, w.d, w.Cq, w.Ck, iters=iters, exact_frac=exact, sample_frac=sample,
                           seed=7, layer=0)
        ws = torch.empty(ig.workspace_size(p), dtype=torch.uint8, device=dev)
        O = torch.empty_like(Q)
        kw = {} if init is None else dict(cq_init=init[0], ck_init=init[1])
        for _ in range(2):
            ig.forward(Q, K, V, p, workspace=ws, out=O, **kw)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(3):
            ig.forward(Q, K, V, p, workspace=ws, out=O, **kw)
        e1.record()
        torch.cuda.synchronize()
        ig.device_status()
        err = float((O.float() - D).pow(2).sum().sqrt()) / dn
        it = ig.forward_intermediates(ws, p)
        return e0.elapsed_time(e1) / 3, err, (it["cq"].clone(), it["ck"].clone())

    for ex, sa in ((0.04, 0.04), (0.08, 0.08), (0.16, 0.16), (0.32, 0.32), (0.08, 0.0), (0.16, 0.0),
                   (0.32, 0.0), (0.64, 0.0)):
        ms, err, _ = run(ex, sa)
        print(json.dumps({"workload": w.name, "exact_frac": ex, "sample_frac": sa, "ms_per_call": round(ms, 3),
                          "rel_l2_vs_dense": round(err, 4), "kmeans_iters": w.iters}))
    ms, err, cent = run(0.16, 0.16)
    ms_w, err_w, _ = run(0.16, 0.16, iters=2, init=cent)
    print(json.dumps({"workload": w.name, "exact_frac": 0.16, "sample_frac": 0.16, "cold_ms": round(ms, 3),
                      "cold_rel_l2": round(err, 4), "cold_iters": w.iters, "warm_ms": round(ms_w, 3),
                      "warm_rel_l2": round(err_w, 4), "warm_iters": 2,
                      "warm_init": "centroids of the previous call on the same inputs"}))


if __name__ == "__main__":
    sys.exit(main())
