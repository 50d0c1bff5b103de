#!/usr/bin/env python
"""ADA paged decode benchmark: KV tokens.heads/s on B200 and the fraction of
the HBM roofline, next to a dense bf16 paged-decode baseline on the same box.

Default workload: the 128K long-context decode (B=1, T=131072, 32 query /
8 KV heads, d=128, P=64, budget 40% of the dense fp16 KV bytes, the first 64
and last 1024 tokens protected, Zipf(1.1) utilities).  One step = one
skv_decode_attention call (decode kernel + merge kernel) over the whole
resident store.  Steps run as CUDA-graph replays so that host launch cost
does not enter the device timeline; two copies of the store alternate so the
~215 MB read per step never comes from L2 (126 MB).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl skv|reference]

Under torchrun each rank (one GPU) decodes its own copy of the workload
(independent sequences: weak scaling, no collective on the data path); the
step time is the max over ranks.  `--gpus N` must match the launcher's
WORLD_SIZE (a mismatch exits with status 2); without a launcher, N > 1
re-runs the command under torch.distributed.run with N local processes.  --impl reference times the CPU oracle on a
bounded sample of the same workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ADA decode KV tokens·heads/s at 1 B200; achieved HBM GB/s as % of peak"
UNIT = "KV tokens·heads/s"
TIER_BYTES = (512, 196, 180)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="skv", choices=["skv", "reference"])
    ap.add_argument("--seq-len", type=int, default=131072)
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--no-dense", action="store_true", help="skip the dense bf16 baseline")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline leg")
    ap.add_argument("--no-append", action="store_true", help="skip the skv_append timing")
    ap.add_argument("--no-t0-bf16", action="store_true",
                    help="skip the fused T0 / bf16 variant's timing")
    ap.add_argument("--no-retier", action="store_true",
                    help="skip the skv_retier timing (it follows the append leg)")
    ap.add_argument("--no-utility", action="store_true",
                    help="skip the skv_decode_utility timing")
    ap.add_argument("--cp", action="store_true",
                    help="context-parallel decode: the ranks share one sequence, each "
                         "holding a slice of its positions (strong scaling)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (Llama layer, ragged batch, 32-layer "
                         "pipeline, tiny)")
    ap.add_argument("--graph-steps", type=int, default=100)
    ap.add_argument("--seed", type=int, default=0)
    return ap.parse_args()


def workload_desc(T):
    return (f"long_context: B=1, T={T}, 32 query / 8 KV heads (GQA 4), d=128, P=64, "
            f"budget 40% of dense fp16 KV, protect first 64 + last 1024, Zipf(1.1) utility, "
            f"bf16 q")


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.gpu = gpu_index
        self.period = period_ms
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", str(self.period)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self._t.join(timeout=2)
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), util=float(f[4]),
                                 hw=f[6], hwt=f[7], swt=f[8], swp=f[9]))
            except ValueError:
                continue
        load = [r for r in rows if r["util"] >= 50] or rows
        if not load:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        reasons = set()
        for r in load:
            if r["hw"] == "Active":
                reasons.add("hw_slowdown")
            if r["hwt"] == "Active":
                reasons.add("hw_thermal_slowdown")
            if r["swt"] == "Active":
                reasons.add("sw_thermal_slowdown")
            if r["swp"] == "Active":
                reasons.add("sw_power_cap")
        return {"sm_mhz": float(np.median([r["sm"] for r in load])),
                "sm_max_mhz": max(r["smax"] for r in load), "reasons": sorted(reasons),
                "samples": len(load)}


# ----------------------------------------------------------------- helpers --

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def split_costs(payload):
    """The decode's split weight per tier (the library's rule): a page's
    payload bytes, a T2 page at least a T1 page's."""
    p0, p1, p2 = (int(x) for x in payload)
    return [p0, p1, max(p2, p1)]


def written_partials(indptr: np.ndarray, ids: np.ndarray, payload, S: int) -> int:
    """(run, unit) partials the decode kernel writes (and the merge kernel
    reads back).  Pages cost their tier's split weight (split_costs).  With at most S
    units, unit u gets runs [B(u), B(u+1)), B(u) = u + round(P(u)(S-U)/C)
    (P(u) the bytes before u, C the total) when S >= 8 U; otherwise page g is in run
    floor(C(g) S / C), C(g) the bytes before it.  A unit spread over several
    runs gets one partial per run, a unit inside one run none."""
    N = int(indptr[-1])
    U = len(indptr) - 1
    if N == 0:
        return 0
    cost = np.asarray(split_costs(payload), np.int64)[np.asarray(ids[:N], np.uint32) >> 30]
    before = np.concatenate([[0], np.cumsum(cost)[:-1]])
    total = int(cost.sum())
    n = 0
    if 8 * U <= S:  # unit-aligned split: at least 8 runs per unit
        ucost = [int(cost[int(indptr[u]):int(indptr[u + 1])].sum()) for u in range(U)]
        P = np.concatenate([[0], np.cumsum(ucost)])
        first = [u + (2 * int(P[u]) * (S - U) + total) // (2 * total) for u in range(U + 1)]
        for u in range(U):
            k = first[u + 1] - first[u]
            n += k if (k > 1 and ucost[u] > 0) else 0
        return n
    run = np.array([(int(x) * S) // total for x in before], np.int64)
    for u in range(U):
        a, b = int(indptr[u]), int(indptr[u + 1])
        k = len(np.unique(run[a:b])) if b > a else 0
        n += k if k > 1 else 0
    return n


def max_over_ranks(elapsed_ms: float, device) -> float:
    """The max over ranks of a device-timed region (every rank gets it); the
    value itself on a single process."""
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return elapsed_ms
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(units_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank decodes its own store of
    units_per_rank token-heads per step (weak scaling, no exchange)."""
    return world * units_per_rank / (ms_per_step * 1e-3)


def clone_cache(cache):
    from long_context_decode_ada_b200 import skv
    c2 = skv.PagedCache(cache.ctx, cache.B, cache.Hkv, cache.Tmax, cache.pool_slots,
                        page_cap=cache.page_cap, device=cache.device)
    for t in range(3):
        c2.pools[t].copy_(cache.pools[t])
    c2.page_indptr.copy_(cache.page_indptr)
    c2.page_tier_indptr.copy_(cache.page_tier_indptr)
    c2.page_ids.copy_(cache.page_ids)
    c2.tier.copy_(cache.tier)
    return c2


def timed_graph_steps(step_fns, steps, warmup, graph_steps, stream, mid_events=None):
    """Warm up eagerly, then capture two CUDA graphs of `graph_steps` steps:
    the timed one (the steps alone, nothing between them) and a profile one
    whose steps carry events (before the step, after its decode kernel,
    after the step).  Returns (timed graph, tail graph for steps %
    graph_steps, profile graph, its event triples, replays of the timed
    graph that make `steps`)."""
    for i in range(warmup):
        step_fns[i % len(step_fns)](None)
    torch.cuda.synchronize()
    gsteps = max(1, min(graph_steps, steps))
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(gsteps)]
    for e3 in ev:                 # torch creates the CUDA events on first record
        for e in e3:
            e.record()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(gsteps):
            step_fns[i % len(step_fns)](None)
    g_prof = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_prof):
        for i in range(gsteps):
            ev[i][0].record()
            step_fns[i % len(step_fns)](ev[i][1])
            ev[i][2].record()
    tail = steps % gsteps
    g_tail = None
    if tail:
        g_tail = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_tail):
            for i in range(tail):
                step_fns[i % len(step_fns)](None)
    g.replay()
    g_prof.replay()
    torch.cuda.synchronize()
    return g, g_tail, g_prof, ev, steps // gsteps


# ------------------------------------------------------------- main (skv) --

def run_skv(args, rank, world, local_rank):
    from long_context_decode_ada_b200 import skv
    from long_context_decode_ada_b200 import workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    T = args.seq_len
    t_gen = time.time()
    w = wl.long_context(seed=args.seed + 1000 * rank, T=T)
    t_gen = time.time() - t_gen
    ctx = skv.Context(w.P)
    d = skv.workload_to_device(w, dev)

    # ---- ingest: allocate + encode (off the decode path; timed for context,
    # warm: the first pass loads the kernels' modules)
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    cache = skv.PagedCache(ctx, w.B, w.Hkv, w.Tmax, w.pool_slots, device=dev)
    cache.allocate(d["K"], d["seq_lens"], d["utility"], d["protect"], w.mode, d["budget"],
                   d["quota"], d["free_lists"])
    cache.encode(d["K"], d["V"], d["seq_lens"])
    torch.cuda.synchronize()
    e0.record()
    cache.allocate(d["K"], d["seq_lens"], d["utility"], d["protect"], w.mode, d["budget"],
                   d["quota"], d["free_lists"])
    e1.record()
    cache.encode(d["K"], d["V"], d["seq_lens"])
    e2.record()
    cache.check()
    alloc_ms, enc_ms = e0.elapsed_time(e1), e1.elapsed_time(e2)
    caches = [cache, clone_cache(cache)]

    tier_counts = torch.bincount(cache.tier.flatten().to(torch.int64), minlength=4).cpu().numpy()
    indptr = cache.page_indptr.cpu().numpy()
    n_pages = int(indptr[-1])
    ids = cache.page_ids[:n_pages].cpu().numpy().view(np.uint32)
    pages_per_tier = np.bincount(ids >> 30, minlength=3)
    resident = int(tier_counts[:3].sum())            # kept (seq, kv head, token) triples
    sm_count, default_splits = ctx.device_info()
    S = args.num_splits or default_splits
    G = w.Hq // w.Hkv
    nparts = written_partials(indptr, ids, caches[0].payload, S)
    q_bytes = w.B * w.Hq * 128 * 2
    algo_bytes = (int(sum(int(tier_counts[t]) * TIER_BYTES[t] for t in range(3)))
                  + 16 * n_pages + 4 * n_pages + 4 * len(indptr) + q_bytes
                  + nparts * G * 132 * 4)
    payload_bytes = int(sum(int(pages_per_tier[t]) * caches[0].payload[t] for t in range(3)))

    stream = torch.cuda.current_stream()
    ws = [c.workspace(w.Hq, S) for c in caches]
    # out and lse in one buffer (lse right after out): the host step then
    # returns both in one copy
    nrow = w.B * w.Hq
    res = torch.empty(nrow * 129, dtype=torch.float32, device=dev)
    out, lse = res[:nrow * 128].view(w.B, w.Hq, 128), res[nrow * 128:].view(w.B, w.Hq)

    def make_step(c, wsp):
        def step(mid_event):
            ctx.set_profile_event(mid_event)
            c.decode(d["q"], d["q_dtype"], w.Hq, out=out, lse=lse, workspace=wsp, num_splits=S)
        return step

    step_fns = [make_step(caches[0], ws[0]), make_step(caches[1], ws[1])]
    g, g_tail, g_prof, ev, reps = timed_graph_steps(step_fns, args.steps, args.warmup,
                                                    args.graph_steps, stream)
    ctx.set_profile_event(None)
    caches[0].check()

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(reps):
        g.replay()
    if g_tail is not None:
        g_tail.replay()
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    elapsed_ms = t0.elapsed_time(t1)
    caches[0].check()
    elapsed_ms = max_over_ranks(elapsed_ms, dev)
    ms_per_step = elapsed_ms / args.steps
    value = whole_job_value(resident, world, ms_per_step)
    # the decode kernel's own duration: the profile graph, after the timed region
    g_prof.replay()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(c) for a, b, c in ev]
    kern_ms = [a.elapsed_time(b) for a, b, c in ev]
    kern_ms_avg = float(np.mean(kern_ms))
    peak, peak_kind = measured_peaks()
    achieved = algo_bytes / (kern_ms_avg * 1e-3) / 1e9

    # ---- end to end: host q -> device, decode, out/lse -> host, every step
    e2e = None
    if rank == 0 or world > 1:
        q_host = d["q"].cpu().pin_memory()
        res_host = torch.empty(nrow * 129, dtype=torch.float32).pin_memory()
        out_host = res_host[:nrow * 128].view(w.B, w.Hq, 128)
        lse_host = res_host[nrow * 128:].view(w.B, w.Hq)
        scratch = (torch.empty_like(d["q"]), res, None)   # packed: out then lse
        e2e_steps = max(10, min(args.steps, 2000))
        # a stream of its own (the legacy default stream's implicit
        # synchronisation costs about 4 us a step)
        es = torch.cuda.Stream(device=dev)
        for i in range(5):
            caches[i % 2].decode_host(q_host, d["q_dtype"], w.Hq, res_host, None, scratch,
                                      workspace=ws[i % 2], num_splits=S, stream=es)
        ta = time.perf_counter()
        for i in range(e2e_steps):
            caches[i % 2].decode_host(q_host, d["q_dtype"], w.Hq, res_host, None, scratch,
                                      workspace=ws[i % 2], num_splits=S, stream=es)
        e2e_host_call_ms = (time.perf_counter() - ta) * 1e3 / e2e_steps
        caches[0].check()
        # the pipelined host step: call k issues step k and waits for step
        # k - 1 (two alternating host buffer sets); every step still copies
        # its q in and its out + lse + error word out
        sets = [(d["q"].cpu().pin_memory(), torch.empty(nrow * 129, dtype=torch.float32)
                 .pin_memory()) for _ in range(2)]
        q_dev2 = torch.empty(2 * d["q"].numel(), dtype=d["q"].dtype, device=dev)  # two slots
        res2 = torch.empty(2 * nrow * 129, dtype=torch.float32, device=dev)
        for i in range(5):
            caches[i % 2].decode_host_pipelined(sets[i % 2][0], d["q_dtype"], w.Hq,
                                                sets[i % 2][1], q_dev2, res2, workspace=ws[i % 2],
                                                num_splits=S, stream=es)
        ctx.drain_host_steps()
        ta = time.perf_counter()
        for i in range(e2e_steps):
            caches[i % 2].decode_host_pipelined(sets[i % 2][0], d["q_dtype"], w.Hq,
                                                sets[i % 2][1], q_dev2, res2, workspace=ws[i % 2],
                                                num_splits=S, stream=es)
        ctx.drain_host_steps()
        e2e_ms = (time.perf_counter() - ta) * 1e3 / e2e_steps
        breakdown = e2e_breakdown(caches, ws, d, w, q_host, res_host, res, out, lse, S, es,
                                  e2e_steps)
        e2e = {"value": world * resident / (e2e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": int(q_host.numel() * q_host.element_size()),
               "d2h_bytes_per_step": int(out_host.numel() * 4 + lse_host.numel() * 4 + 4),
               "ms_per_step": e2e_ms, "steps": e2e_steps,
               "host_call_ms_per_step": e2e_host_call_ms, "breakdown": breakdown,
               "how": "skv_decode_attention_host_pipelined every step (call k issues step k "
                      "and waits for step k - 1; two alternating pinned buffer sets): pinned "
                      "host q -> device on a copy stream, the decode on a stream of its own, "
                      "out + lse (packed, one copy) and the error word -> pinned host on a "
                      "second copy stream; host wall clock over all steps and the final drain. "
                      "host_call_ms_per_step: the unpipelined skv_decode_attention_host (one "
                      "synchronous call a step)"}

    # ---- dense bf16 paged-decode baseline on the same K/V
    dense = None
    if not args.no_dense:
        n_dense = w.B * w.Hkv * (-(-T // w.P))
        dcs = []
        for k in range(2):
            dc = skv.DenseCache(ctx, w.B, w.Hkv, w.Tmax, n_dense, device=dev)
            dc.pack(d["K"], d["V"], d["seq_lens"], torch.arange(n_dense, dtype=torch.int32))
            dc.check()
            dcs.append(dc)
        dws = [dc.workspace(w.Hq, S) for dc in dcs]

        def dstep(i):
            def f(mid):
                ctx.set_profile_event(mid)
                dcs[i].decode(d["q"], d["q_dtype"], w.Hq, out=out, lse=lse, workspace=dws[i],
                              num_splits=S)
            return f
        dsteps = max(10, min(args.steps, 2000))
        gd, gd_tail, gd_prof, evd, repd = timed_graph_steps([dstep(0), dstep(1)], dsteps,
                                                            min(args.warmup, 20), args.graph_steps,
                                                            stream)
        ctx.set_profile_event(None)
        torch.cuda.synchronize()
        ta, tb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ta.record()
        for _ in range(repd):
            gd.replay()
        if gd_tail is not None:
            gd_tail.replay()
        tb.record()
        torch.cuda.synchronize()
        gd_prof.replay()
        torch.cuda.synchronize()
        dcs[0].check()
        dms = ta.elapsed_time(tb) / dsteps
        dk = float(np.mean([a.elapsed_time(b) for a, b, c in evd]))
        dbytes = w.B * w.Hkv * T * 512 + 16 * n_dense + 4 * n_dense
        dense = {"value": world * w.B * w.Hkv * T / (dms * 1e-3), "unit": UNIT + " (all tokens)",
                 "ms_per_step": dms, "kernel_ms": dk,
                 "achieved_gbs": dbytes / (dk * 1e-3) / 1e9,
                 "frac": dbytes / (dk * 1e-3) / 1e9 / peak,
                 "ada_speedup_step": dms / ms_per_step}
        del dcs, dws

    # ---- the fused T0 / bf16 variant: the same tiers with T0 pages in bf16,
    # decoded on the bf16 path, timed as the main step
    t0b = None
    if not args.no_t0_bf16:
        ctx_b = skv.Context(w.P, t0_bf16=True)
        bcs = []
        for k in range(2):
            bc = skv.PagedCache(ctx_b, w.B, w.Hkv, w.Tmax, w.pool_slots, device=dev)
            bc.allocate(d["K"], d["seq_lens"], d["utility"], d["protect"], w.mode, d["budget"],
                        d["quota"], d["free_lists"])
            bc.encode(d["K"], d["V"], d["seq_lens"])
            bc.check()
            bcs.append(bc)
        bws = [bc.workspace(w.Hq, S) for bc in bcs]

        def bstep(i):
            def f(mid):
                ctx_b.set_profile_event(mid)
                bcs[i].decode(d["q"], d["q_dtype"], w.Hq, out=out, lse=lse, workspace=bws[i],
                              num_splits=S)
            return f
        bsteps = max(10, min(args.steps, 2000))
        gb, gb_tail, gb_prof, evb, repb = timed_graph_steps([bstep(0), bstep(1)], bsteps,
                                                            min(args.warmup, 20), args.graph_steps,
                                                            stream)
        ctx_b.set_profile_event(None)
        torch.cuda.synchronize()
        ta, tb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ta.record()
        for _ in range(repb):
            gb.replay()
        if gb_tail is not None:
            gb_tail.replay()
        tb.record()
        torch.cuda.synchronize()
        gb_prof.replay()
        torch.cuda.synchronize()
        bcs[0].check()
        bms = ta.elapsed_time(tb) / bsteps
        bk = float(np.mean([a.elapsed_time(b) for a, b, c in evb]))
        t0b = {"ms_per_step": bms, "kernel_ms": bk, "steps": bsteps,
               "step_ratio_vs_mixed": bms / ms_per_step,
               "kernel_ratio_vs_mixed": bk / kern_ms_avg,
               "how": "the same tiers and bytes, T0 pages in bf16 decoded on the dense "
                      "kernel's bf16 logit and P.V steps (skv_config.t0_bf16); graph replays "
                      "over two stores, CUDA events"}
        del bcs, bws, gb, gb_tail, gb_prof

    # ---- the decode with the utility update (skv_decode_utility) on the same
    # two stores, timed as the main step (graph replays, CUDA events)
    utility = None
    if not args.no_utility:
        uts = [torch.zeros((w.B, w.Hkv, w.Tmax), dtype=torch.float32, device=dev)
               for _ in range(2)]
        uws = [c.utility_workspace(w.Hq, S) for c in caches]

        def make_ustep(k):
            def step(mid_event):
                ctx.set_profile_event(mid_event)
                caches[k].decode_utility(d["q"], d["q_dtype"], w.Hq, d["seq_lens"], uts[k], 0.9,
                                         out=out, lse=lse, workspace=uws[k], num_splits=S)
            return step

        u_steps = max(2, min(1000, args.steps))
        gu, gu_tail, gu_prof, evu, reps_u = timed_graph_steps(
            [make_ustep(0), make_ustep(1)], u_steps, 5, args.graph_steps, stream)
        ctx.set_profile_event(None)
        ua, ub = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ua.record()
        for _ in range(reps_u):
            gu.replay()
        if gu_tail is not None:
            gu_tail.replay()
        ub.record()
        torch.cuda.synchronize()
        caches[0].check()
        gu_prof.replay()
        torch.cuda.synchronize()
        u_kern = float(np.mean([a.elapsed_time(b) for a, b, c in evu]))
        u_rest = float(np.mean([b.elapsed_time(c) for a, b, c in evu]))
        G = w.Hq // w.Hkv
        logit_bytes = resident * G * 4
        utility = {"us_per_step": ua.elapsed_time(ub) * 1e3 / u_steps, "steps": u_steps,
                   "decode_kernel_us": u_kern * 1e3, "merge_and_update_us": u_rest * 1e3,
                   "plain_step_us": ms_per_step * 1e3,
                   "logit_bytes_written": logit_bytes,
                   "update_bytes": logit_bytes + w.B * w.Hkv * w.Tmax * (1 + 4 + 4 + 4),
                   "how": "skv_decode_utility (decode with per-row logit capture, merge, "
                          "utility update u <- 0.9 u + mass) in graphs of "
                          f"{min(args.graph_steps, u_steps)} steps over the two stores; the "
                          "profile graph's events split the decode kernel from the rest"}
        del uts, uws, gu, gu_tail, gu_prof

    # ---- decode-time append (skv_append) on the same recipe: a store built
    # n_app tokens short; the first n_eager appends timed one after another,
    # then the serving step (append + decode, one CUDA graph) for the rest
    append = None
    retier = None
    serving = None
    if not args.no_append:
        import dataclasses
        n_app, n_eager = 128, 64
        wa = dataclasses.replace(w, seq_lens=(w.seq_lens - n_app).astype(np.int32))
        slots = list(w.pool_slots)
        slots[0] += w.B * w.Hkv * (n_app // w.P + 2)
        # room for the re-tiering's rewritten pages (the window's T0 pages from
        # the first demoted row on, the last T1 / T2 pages and new ones)
        slots = [x + w.B * w.Hkv * (1024 // w.P + 4) for x in slots]
        wa = dataclasses.replace(wa, pool_slots=slots,
                                 free_lists=[np.arange(x, dtype=np.uint32) for x in slots])
        da = skv.workload_to_device(wa, dev)
        ca = skv.build_cache(ctx, wa, da)
        ca.check()
        seq_a = da["seq_lens"].clone()
        kv = [(d["K"][:, :, T - n_app + i].contiguous(), d["V"][:, :, T - n_app + i].contiguous())
              for i in range(n_app)]
        ca.append(*kv[0], seq_a)      # allocates the append workspace
        torch.cuda.synchronize()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record()
        for i in range(1, n_eager):
            ca.append(*kv[i], seq_a)
        eb.record()
        torch.cuda.synchronize()
        ca.check()
        append = {"us_per_step": ea.elapsed_time(eb) * 1e3 / (n_eager - 1), "steps": n_eager - 1,
                  "how": "skv_append of one token per sequence and kv head, eager launches "
                         "(3 kernels each; pages are added every P steps), CUDA events "
                         "around the steps"}
        # ---- the serving step: skv_append of the new token (its K / V in the
        # step's input buffers, where the model would write them) and the
        # decode over the store it grew, 8 steps to a CUDA graph
        per_graph = 8
        kvb = [(kv[n_eager + j][0].clone(), kv[n_eager + j][1].clone()) for j in range(per_graph)]
        wsa = [ca.workspace(w.Hq, S) for _ in range(2)]
        out_s = torch.empty_like(out)
        lse_s = torch.empty_like(lse)
        gs = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gs):
            for j in range(per_graph):
                ca.append(*kvb[j], seq_a)
                ca.decode(d["q"], d["q_dtype"], w.Hq, out=out_s, lse=lse_s, workspace=wsa[j % 2],
                          num_splits=S)
        torch.cuda.synchronize()
        n_srv = (n_app - n_eager) // per_graph * per_graph
        ea.record()
        for i in range(n_srv // per_graph):
            gs.replay()
        eb.record()
        torch.cuda.synchronize()
        ca.check()
        assert int(seq_a[0]) == T - (n_app - n_eager - n_srv), "the serving steps appended"
        serving = {"us_per_step": ea.elapsed_time(eb) * 1e3 / n_srv, "steps": n_srv,
                   "how": "per token: skv_append (its K and V in the step's input buffers) and "
                          "the decode over the store it grew, 8 steps to a CUDA graph (the "
                          "buffers hold the same 8 tokens at each replay); 128K store, its last "
                          "64 tokens; CUDA events around the replays"}
        del gs
        # ---- the window roll that follows: the oldest n_app - 1 rows of the
        # protected recent window re-tiered under the budget grown with the
        # appended tokens (skv_retier), on the store the appends left
        if not args.no_retier:
            lo = T - 1024
            demote = torch.zeros((w.B, w.Hkv, w.Tmax), dtype=torch.uint8, device=dev)
            demote[:, :, lo:lo + n_app - 1] = 1
            budget = da["budget"] + int(0.4 * n_app * w.Hkv * 512)
            # warm-up: a re-tiering with nothing demoted (and room in the
            # budget) changes no byte, and loads the kernels' modules
            ca.retier(da["utility"], torch.zeros_like(demote), 2 * budget, seq_a)
            torch.cuda.synchronize()
            ca.check()
            before = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n_pages0 = int(ca.page_indptr[-1])
            cur0 = ca.free_cursor().clone()
            before[0].record()
            released, n_rel = ca.retier(da["utility"], demote, budget, seq_a)
            before[1].record()
            torch.cuda.synchronize()
            ca.check()
            new_t = ca.tier[:, :, lo:lo + n_app - 1].flatten().to(torch.int64)
            retier = {"us": before[0].elapsed_time(before[1]) * 1e3,
                      "rows_demoted": int(w.B * w.Hkv * (n_app - 1)),
                      "demoted_to": {k: int((new_t == i).sum()) for i, k in
                                     enumerate(("T0", "T1", "T2", "dropped"))},
                      "pages_before": n_pages0, "pages_after": int(ca.page_indptr[-1]),
                      "pages_rewritten": int((ca.free_cursor() - cur0).sum()),
                      "pages_released": int(n_rel.item()),
                      "how": "skv_retier of the window's oldest rows after the appends, one "
                             "eager call (snapshot copies, key, select, tier, count, row-map, "
                             "diff, plan, page-write, release and transcode kernels), CUDA "
                             "events around it"}
        del ca, da

    configs = None
    if not args.no_configs:
        del caches, ws
        torch.cuda.empty_cache()
        configs = run_configs(ctx, dev, peak, S_default=default_splits)

    cpu = None
    if rank == 0 and not args.no_cpu:
        cpu = cpu_baseline(T_sample=args.seq_len)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic",
            "config": {"workload": workload_desc(T),
                       "l2": "inputs larger than L2: two rotating copies of the ~215 MB store",
                       "num_splits": S, "graph_steps": args.graph_steps,
                       "resident_tokens_heads": resident,
                       "tier_tokens": {"T0": int(tier_counts[0]), "T1": int(tier_counts[1]),
                                       "T2": int(tier_counts[2]), "dropped": int(tier_counts[3])},
                       "pages": {"T0": int(pages_per_tier[0]), "T1": int(pages_per_tier[1]),
                                 "T2": int(pages_per_tier[2])},
                       "parallelism": f"{world} independent replicas (one per GPU)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(),
                         "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)",
                         "kernel": "decode_kernel<4,false,false,0>", "kernel_ms": kern_ms_avg,
                         "kernel_timing": "serialised launch: `frac` divides by the kernel timed "
                                          "alone (events around it in a profile graph keep the next "
                                          "step from starting early); in the timed graph each "
                                          "step's decode starts while the previous step finishes, "
                                          "so kernel_ms > ms_per_step and `frac_per_step` is the "
                                          "same bytes over the overlapped step time",
                         "achieved_per_step": algo_bytes / (ms_per_step * 1e-3) / 1e9,
                         "frac_per_step": algo_bytes / (ms_per_step * 1e-3) / 1e9 / peak,
                         "algorithmic_bytes": algo_bytes, "payload_bytes_streamed": payload_bytes,
                         "no_reconstruction": no_reconstruction(algo_bytes, nparts, G, w.B * w.Hq,
                                                                 tier_counts)},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": 2 * args.steps,  # decode_kernel + decode_merge_kernel per step
            "clocks": clocks,
            "dense_bf16_baseline": dense,
            "t0_bf16_variant": t0b,
            "ingest": {"allocate_ms": alloc_ms, "encode_ms": enc_ms, "gen_s": t_gen},
            "append": append,
            "serving_step": serving,
            "retier": retier,
            "utility": utility,
            "configs": configs,
            "step_ms_graph_events": float(np.mean(step_ms)),
        }
        print(json.dumps(line), flush=True)


def e2e_breakdown(caches, ws, d, w, q_host, res_host, res, out, lse, S, stream, steps):
    """Where an end-to-end step's time goes.  Per round: an eager
    device-buffer decode (decode + merge) between CUDA events; the result
    copies alone (out + lse packed in one copy, the error word) between
    events; and one skv_decode_attention_host call on the host wall clock.
    The call's time beyond the two device parts is the q copy, host launch
    and the stream-sync wake-up."""
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    scratch = (torch.empty_like(d["q"]), res, None)
    err_host = torch.zeros(1, dtype=torch.int32).pin_memory()
    dec = cop = wall = 0.0
    n = max(10, min(steps, 500))
    for i in range(n + 5):
        c = caches[i % 2]
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            c.decode(d["q"], d["q_dtype"], w.Hq, out=out, lse=lse, workspace=ws[i % 2],
                     num_splits=S, stream=stream)
            ev[1].record(stream)
            res_host.copy_(res, non_blocking=True)
            err_host.copy_(c.err, non_blocking=True)
            ev[2].record(stream)
        stream.synchronize()
        ta = time.perf_counter()
        c.decode_host(q_host, d["q_dtype"], w.Hq, res_host, None, scratch, workspace=ws[i % 2],
                      num_splits=S, stream=stream)
        tb = time.perf_counter()
        if i >= 5:
            wall += tb - ta
            dec += ev[0].elapsed_time(ev[1])
            cop += ev[1].elapsed_time(ev[2])
    dec_us, cop_us, wall_us = dec / n * 1e3, cop / n * 1e3, wall / n * 1e6
    return {"eager_decode_and_merge_us": dec_us, "result_copies_us": cop_us,
            "call_wall_us": wall_us, "q_copy_launch_and_sync_us": wall_us - dec_us - cop_us,
            "steps": n,
            "how": "per round: an eager device-buffer decode between CUDA events, the result "
                   "copies alone between events, and one skv_decode_attention_host call on the "
                   "host wall clock, on the e2e leg's stream; the rest = call - decode - "
                   "copies"}


def store_stats(cache):
    """Tier counts, pages per tier and the decode's algorithmic bytes of one
    store (tier bytes of the resident token-heads + 20 B per page)."""
    tc = torch.bincount(cache.tier.flatten().to(torch.int64), minlength=4).cpu().numpy()
    indptr = cache.page_indptr.cpu().numpy()
    n = int(indptr[-1])
    ids = cache.page_ids[:n].cpu().numpy().view(np.uint32)
    ppt = np.bincount(ids >> 30, minlength=3)
    byt = int(sum(int(tc[t]) * TIER_BYTES[t] for t in range(3))) + 20 * n + 4 * len(indptr)
    return {"tier_tokens": {"T0": int(tc[0]), "T1": int(tc[1]), "T2": int(tc[2]),
                            "dropped": int(tc[3])},
            "pages": {"T0": int(ppt[0]), "T1": int(ppt[1]), "T2": int(ppt[2])},
            "resident_tokens_heads": int(tc[:3].sum()), "bytes": byt}


def graph_time_ms(fns, reps_per_graph, replays):
    """Mean device time of one call of fns (cycled) in CUDA-graph replays:
    3 eager warm-up calls, one graph of reps_per_graph calls, replays timed
    with events on the current stream."""
    for i in range(3):
        fns[i % len(fns)]()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps_per_graph):
            fns[i % len(fns)]()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / (replays * reps_per_graph)


def run_configs(ctx, dev, peak, S_default):
    """The other workloads of the decode path, drawn on the GPU with the same
    recipes: the Llama-3-8B-shaped layer, the ragged batch of 64 (scattered
    pages), the tiny all-T2 store and the 32-layer pipeline (allocate +
    encode per layer, then a decode step over all 32 layers).  Stores larger
    than L2 alternate between two copies; the tiny store (0.7 MB) is timed
    warm in L2 and says so."""
    from long_context_decode_ada_b200 import skv
    from long_context_decode_ada_b200 import workloads as wl
    res = {}

    def one_layer(name, w, copies, note):
        d = skv.workload_to_device(w, dev)
        c0 = skv.build_cache(ctx, w, d)
        c0.check()
        caches = [c0] + [clone_cache(c0) for _ in range(copies - 1)]
        del d["K"], d["V"]
        wss = [c.workspace(w.Hq) for c in caches]
        out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=dev)
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
        fns = [(lambda c=c, wsp=wsp: c.decode(d["q"], d["q_dtype"], w.Hq, out=out, lse=lse,
                                              workspace=wsp)) for c, wsp in zip(caches, wss)]
        ms = graph_time_ms(fns, 20 * copies if copies > 1 else 20, 10)
        c0.check()
        st = store_stats(c0)
        gbs = st["bytes"] / (ms * 1e-3) / 1e9
        res[name] = dict(st, us_per_decode=ms * 1e3, achieved_gbs=gbs, frac=gbs / peak,
                         value=st["resident_tokens_heads"] / (ms * 1e-3), unit=UNIT,
                         B=w.B, Hq=w.Hq, Hkv=w.Hkv, P=w.P, note=note)
        del caches, wss, fns
        torch.cuda.empty_cache()

    one_layer("llama_layer", wl.llama_layer(device=dev), 2,
              "B=8, T=32768, 32q/8kv, P=64, quota 10/50/25/15%; two alternating stores")
    one_layer("ragged_batch", wl.ragged_batch(device=dev), 2,
              "B=64, T~U[1024,8192], P=16, quota 20/40/40/0%, scattered pages; two "
              "alternating stores")
    one_layer("tiny_all_t2", wl.tiny(), 1,
              "B=1, one head, T=4096, P=16, all T2: 0.74 MB, timed warm (in L2)")

    # ---- 32-layer pipeline: allocate + encode per layer, one decode step over all layers
    L = 32
    caches, qs, wss = [], [], []
    alloc_ms = enc_ms = 0.0
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for layer in range(L):
        w = wl.pipeline_layer(layer, device=dev)
        d = skv.workload_to_device(w, dev)
        c = skv.PagedCache(ctx, w.B, w.Hkv, w.Tmax, w.pool_slots, device=dev)
        e[0].record()
        c.allocate(d["K"], d["seq_lens"], d["utility"], d["protect"], w.mode, d["budget"],
                   d["quota"], d["free_lists"])
        e[1].record()
        c.encode(d["K"], d["V"], d["seq_lens"])
        e[2].record()
        c.check()
        alloc_ms += e[0].elapsed_time(e[1])
        enc_ms += e[1].elapsed_time(e[2])
        caches.append(c)
        qs.append(d["q"])
        wss.append(c.workspace(w.Hq))
        del d, w
    Hq = 32
    out = torch.empty((4, Hq, 128), dtype=torch.float32, device=dev)
    lse = torch.empty((4, Hq), dtype=torch.float32, device=dev)

    def step():
        for layer in range(L):
            caches[layer].decode(qs[layer], skv.Q_BF16, Hq, out=out, lse=lse,
                                 workspace=wss[layer])
    ms = graph_time_ms([step], 4, 10)
    for c in caches:
        c.check()
    stats = [store_stats(c) for c in caches]
    byt = sum(s_["bytes"] for s_ in stats)
    tok = sum(s_["resident_tokens_heads"] for s_ in stats)
    tiers = {k: sum(s_["tier_tokens"][k] for s_ in stats) for k in ("T0", "T1", "T2", "dropped")}
    pages = {k: sum(s_["pages"][k] for s_ in stats) for k in ("T0", "T1", "T2")}
    gbs = byt / (ms * 1e-3) / 1e9
    res["pipeline_32_layers"] = {
        "layers": L, "B": 4, "T": 65536, "Hq": 32, "Hkv": 8, "P": 64,
        "allocate_ms_total": alloc_ms, "encode_ms_total": enc_ms,
        "encode_gbs": L * 4 * 8 * 65536 * 512 / (enc_ms * 1e-3) / 1e9,
        "decode_step_us": ms * 1e3, "decode_us_per_layer": ms * 1e3 / L,
        "bytes": byt, "achieved_gbs": gbs, "frac": gbs / peak,
        "value": tok / (ms * 1e-3), "unit": UNIT,
        "tier_tokens": tiers, "pages": pages, "resident_tokens_heads": tok,
        "note": "per layer: outlier channels x20, budget 30% of dense fp16 KV, Zipf(1.2) "
                "utility; allocate and encode timed by events per layer (summed), the decode "
                "step is one graph of 32 decodes (one per layer's store; 10 GB > L2)"}
    del caches, qs, wss
    torch.cuda.empty_cache()
    return res


def _decode_blocks(text: str) -> str:
    """The decode kernel's part of kernels.h: its parameter block and the
    layout of its workspace (the other kernels' blocks do not change it)."""
    out = []
    for head, tail in (("struct DecodeParams {", "\n};"), ("struct DecodeWs {", "return w;\n}")):
        a = text.index(head)
        out.append(text[a:text.index(tail, a) + len(tail)])
    return "\n".join(out)


def decode_source_digest() -> str:
    """sha256 of the decode kernel's sources (decides whether a profiled
    DRAM traffic figure still describes the kernel that runs): decode.cu,
    common.cuh and the decode blocks of kernels.h."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_decode_ada_b200", "csrc")
    for f in ("decode.cu", "common.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(csrc, "kernels.h")) as fh:
        h.update(_decode_blocks(fh.read()).encode())
    return h.hexdigest()


def profile_record():
    """The committed ncu summary of the decode kernel on the 128K store
    (profiles/decode_kernel_long_context.json), or None when the kernel's
    sources changed since it was captured (its digest no longer matches)."""
    path = os.path.join(ROOT, "profiles", "decode_kernel_long_context.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("decode_source_sha256") != decode_source_digest():
        return None
    return rec


def no_reconstruction(algo_bytes, nparts, G, rows, tier_counts):
    """The decode writes no dense key (technical summary 2.1): the bytes the
    kernel's SMs store per launch (ncu: global + local + atomic store
    sectors) against its partials + outputs + 1% of the bytes it streams,
    and against what rebuilding its T1/T2 keys in fp16 would write."""
    rec = profile_record()
    if rec is None:
        return None
    outputs = rows * 128 * 4 + rows * 4 + 8 * rows
    bound = nparts * G * 132 * 4 + outputs + 0.01 * algo_bytes
    return {"sm_store_bytes": rec["sm_store_bytes"], "dram_bytes_write": rec["dram_bytes_write"],
            "bound_bytes": int(bound), "ok": rec["sm_store_bytes"] <= bound,
            "rebuilt_keys_bytes": int(tier_counts[1] + tier_counts[2]) * 256}


def profiled_traffic():
    """dram__bytes_read.sum + dram__bytes_write.sum per decode launch from the
    committed ncu summary, or None when the kernel changed since it was taken."""
    rec = profile_record()
    return None if rec is None else int(rec["traffic_bytes_per_launch"])


# -------------------------------------------------------- oracle (CPU) ----

def cpu_baseline(T_sample: int, min_seconds: float = 10.0):
    """Time the oracle's decode (as it stands) on the host cores on a bounded
    sample of the same workload: the long-context recipe at T_sample tokens,
    decoded repeatedly until at least min_seconds of CPU work have run.  The
    sample's tiers come from the oracle's own allocation."""
    import oracle
    from long_context_decode_ada_b200 import workloads as wl
    w = wl.long_context(seed=1, T=T_sample)
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, w.protect,
                           w.mode, w.budget, w.quota)
    resident = int((tier != 3).sum())
    reps = 0
    t = time.perf_counter()
    while True:
        oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q, w.q_dtype)
        reps += 1
        if time.perf_counter() - t >= min_seconds:
            break
    total = time.perf_counter() - t
    dt = total / reps
    return {"value": resident / dt, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"long_context recipe at T={T_sample} (B=1, 8 KV / 32 query heads, "
                      f"{resident} resident token-heads), oracle decode only, {reps} decodes "
                      f"in {total:.1f} s",
            "seconds": total}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, timed per step on a bounded sample."""
    if rank != 0:
        return
    import oracle
    from long_context_decode_ada_b200 import workloads as wl
    T_sample = 4096
    w = wl.long_context(seed=1, T=T_sample)
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, w.protect,
                           w.mode, w.budget, w.quota)
    resident = int((tier != 3).sum())

    def step():
        oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q, w.q_dtype)

    for _ in range(max(0, min(args.warmup, 3))):
        step()
    steps = args.steps
    t = time.perf_counter()
    budget_s = 120.0
    done = 0
    for i in range(steps):
        step()
        done += 1
        if time.perf_counter() - t > budget_s:
            break
    dt = (time.perf_counter() - t) / done
    value = resident / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": done, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": workload_desc(args.seq_len),
                       "sample": f"each step decodes the long_context recipe at T={T_sample}"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(),
                             "kind": "oracle",
                             "sample": f"long_context recipe at T={T_sample}, {resident} "
                                       f"resident token-heads per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def run_cp(args, rank, world, local_rank):
    """Context-parallel decode of one 128K sequence over the ranks: rank r
    holds slice r of its positions (its own allocate + encode), a step is
    the local decode, the all-gather of the packed partials and the merge.
    Enough copies of each slice's store rotate that the inputs of
    consecutive steps exceed L2."""
    from long_context_decode_ada_b200 import cp, skv
    from long_context_decode_ada_b200 import workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    T = args.seq_len
    w = wl.long_context(seed=args.seed, T=T)          # the same sequence on every rank
    ws = cp.slice_workload(w, world, rank)
    ctx = skv.Context(w.P)
    d = skv.workload_to_device(ws, dev)
    first = skv.build_cache(ctx, ws, d)
    first.check()
    store_bytes = sum(int(p.numel()) for p in first.pools)
    n_copies = max(2, -(-300_000_000 // max(store_bytes, 1)) + 1)
    caches = [first] + [clone_cache(first) for _ in range(n_copies - 1)]
    del d["K"], d["V"]
    torch.cuda.empty_cache()
    S = args.num_splits
    decs = [cp.ContextParallelDecoder(c, w.Hq, num_splits=S) for c in caches]
    resident = int((first.tier != 3).sum().item())
    total = torch.tensor([resident], dtype=torch.int64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(total)
    total = int(total.item())
    stream = torch.cuda.current_stream()

    def make_step(k):
        def step(mid_event):
            ctx.set_profile_event(mid_event)
            decs[k].step(d["q"], d["q_dtype"])   # on the current (capturing) stream
        return step

    g, g_tail, g_prof, ev, reps = timed_graph_steps(
        [make_step(k) for k in range(n_copies)], args.steps, args.warmup,
        min(args.graph_steps, 10 * n_copies), stream)
    ctx.set_profile_event(None)
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(reps):
        g.replay()
    if g_tail is not None:
        g_tail.replay()
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    ms_per_step = max_over_ranks(t0.elapsed_time(t1), dev) / args.steps
    g_prof.replay()
    torch.cuda.synchronize()
    first.check()
    kern = float(np.mean([a.elapsed_time(b) for a, b, c in ev]))
    rest = float(np.mean([b.elapsed_time(c) for a, b, c in ev]))
    del g, g_tail, g_prof      # graphs holding NCCL calls go before the process group
    if rank == 0:
        line = {
            "metric": METRIC, "value": total / (ms_per_step * 1e-3),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": workload_desc(T) + f", context-parallel over {world} ranks "
                                                       f"(slices of {ws.Tmax} positions)",
                       "parallelism": f"cp{world}", "num_splits": S or "default",
                       "l2": f"{n_copies} rotating copies of each rank's "
                             f"{store_bytes / 1e6:.0f} MB store",
                       "resident_tokens_heads": total},
            "cp": {"local_decode_kernel_us": kern * 1e3,
                   "exchange_and_merge_us": rest * 1e3,
                   "how": "graph replays of decode + all-gather + merge steps; the profile "
                          "graph's events split rank 0's local decode kernel from the rest"},
            "gpu_launches": 3 * args.steps,   # decode, its merge, the partials' merge
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def resolve_launch(gpus: int, env, argv):
    """What `--gpus N` means for this process, from the launcher's environment.

    - ("run", world, rank, local_rank): WORLD_SIZE is set and equals N (a
      torchrun rank), or N = 1 without a launcher;
    - ("spawn", cmd): N > 1 and no launcher: re-run this command under
      torch.distributed.run with N processes on this node (127.0.0.1);
    - ("error", message): WORLD_SIZE is set and differs from N, or N < 1.
    The rank count and the reported n_gpus can therefore never disagree."""
    if gpus < 1:
        return ("error", f"--gpus must be >= 1 (got {gpus})")
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != gpus:
            return ("error", f"--gpus {gpus} but the launcher started {world} ranks "
                             f"(WORLD_SIZE={world}); they must agree")
        return ("run", world, int(env.get("RANK", "0")), int(env.get("LOCAL_RANK", "0")))
    if gpus == 1:
        return ("run", 1, 0, 0)
    port = env.get("MASTER_PORT") or "29517"
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__)] + list(argv)
    return ("spawn", cmd)


def main():
    args = parse_args()
    how = resolve_launch(args.gpus, os.environ, sys.argv[1:])
    if how[0] == "error":
        print(f"bench.py: {how[1]}", file=sys.stderr)
        sys.exit(2)
    if how[0] == "spawn":
        sys.exit(subprocess.call(how[1]))
    _, world, rank, local_rank = how
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.cp:
            run_cp(args, rank, world, local_rank)
        else:
            run_skv(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
