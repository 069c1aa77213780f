"""Benchmark: packed-prefix attention fwd+bwd useful TFLOP/s on B200 (and its fraction of the bf16 tensor peak).

One step = the whole hot path over one packed batch: pp_build_meta (position ids + tile schedule), pp_rope (Q, K),
pp_attn_fwd (O, LSE) and pp_attn_bwd (dQ, dK, dV). Useful FLOPs count allowed (query, key) pairs only: 4*d per pair
forward and 10*d per pair backward, per q head. Inputs are synthetic (workloads/), resident in HBM and larger than
L2, so no flush is needed between steps. `e2e` times the same steps through the public API with pinned host buffers:
the host->device copy of q, k, v, dout and the device->host copy of dq, dk, dv are inside its timed region.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload dpo|grpo|longprefix|hetero|tiny]
       python bench.py --impl reference ...   (the fp64 CPU oracle on a bounded sample of the same workload)
Multi-GPU: launched by torch.distributed.run, one rank per GPU; each rank runs its own batch (weak scaling, no
data-path collective); the step time is the max over ranks.
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

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "dpo"
L2_BYTES = 126 * 2 ** 20
KERNEL_SOURCES = ("shared_prefix_packed_b200/csrc",)


def pair_count(P, S):
    tot = 0
    for p, ss in zip(P, S):
        tot += p * (p + 1) // 2 + sum(s * p + s * (s + 1) // 2 for s in ss)
    return tot


def unpacked_pairs(P, S):
    return sum((p + s) * (p + s + 1) // 2 for p, ss in zip(P, S) for s in ss) + sum(
        p * (p + 1) // 2 for p, ss in zip(P, S) if not ss)


# Datasheet dense bf16 tensor peak of one B200: NVIDIA's HGX B200 datasheet lists 36 PFLOPS FP16/BF16 for 8 GPUs
# with 2:4 sparsity, i.e. 18 PFLOPS dense for 8 GPUs, 2.25 PFLOPS dense per GPU.
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_SOURCE = "NVIDIA HGX B200 datasheet: 36 PFLOPS FP16/BF16 per 8 GPUs with 2:4 sparsity = 2.25 dense per GPU"


def unpacked_layout(P, S):
    """The same preference samples without packing: every response becomes its own sequence P || S_i (a group with
    P' = P and one response); a group without responses keeps its prefix alone."""
    Pu, Su = [], []
    for p, ss in zip(P, S):
        if not ss:
            Pu.append(p)
            Su.append([])
        for s_ in ss:
            Pu.append(p)
            Su.append([s_])
    return Pu, Su


def shard_groups(P, S, world):
    """Split one batch's groups across `world` ranks, longest processing time first: groups in decreasing order of
    their allowed pairs (their attention cost), each to the rank with the least cost so far (ties: lowest rank).
    Groups are independent (no attention crosses them), so each rank runs its share with no data-path collective.
    Returns one sorted list of group indices per rank."""
    cost = [pair_count([p], [ss]) for p, ss in zip(P, S)]
    load = [0] * world
    parts = [[] for _ in range(world)]
    for g in sorted(range(len(P)), key=lambda g: (-cost[g], g)):
        r = min(range(world), key=lambda r: (load[r], r))
        parts[r].append(g)
        load[r] += cost[g]
    return [sorted(x) for x in parts]


def flops_of(name, P, S):
    w = W.WORKLOADS[name]
    pairs = pair_count(P, S)
    return pairs, 4 * w.head_dim * pairs * w.num_heads_q, (10 * w.head_dim * pairs * w.num_heads_q
                                                          if w.backward else 0)


def rank_tensor_seed(name, rank):
    """Each rank draws its own batch of the same shape (weak scaling: per-GPU work fixed as N grows)."""
    return W.WORKLOADS[name].tensor_seed + 7919 * rank


def max_over_ranks(value, device, dist=None):
    """Max of a per-rank float over all ranks (the step time the job is charged with)."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank, world, ms_per_step):
    """Whole-job throughput: the useful FLOPs of all ranks over the slowest rank's step time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash():
    h = hashlib.sha256()
    for d in KERNEL_SOURCES:
        base = os.path.join(ROOT, d)
        for fn in sorted(os.listdir(base)):
            with open(os.path.join(base, fn), "rb") as f:
                h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernels, workload):
    """DRAM bytes per launch summed over `kernels`, from the committed ncu summary, if every one of them was taken
    on the current kernel sources and on this workload (None otherwise)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash()
    found = {}
    with open(path) as f:
        for ln in f:
            parts = dict(p.split("=", 1) for p in ln.strip().split() if "=" in p)
            if parts.get("kernel") in kernels and parts.get("sources") == src and parts.get("workload") == workload:
                try:
                    found[parts["kernel"]] = float(parts["dram_bytes_per_launch"])
                except (KeyError, ValueError):
                    return None
    if set(found) != set(kernels):
        return None
    return sum(found.values())


class ClockSampler:
    """nvidia-smi samples (200 ms) while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"pp_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for ln in f:
                c = [x.strip() for x in ln.split(",")]
                if len(c) < 9:
                    continue
                try:
                    sm.append(float(c[1]))
                    mx.append(float(c[2]))
                except ValueError:
                    continue
                for n, v in zip(names, c[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------------- GPU arm
def run_gpu(args):
    import torch
    import torch.distributed as dist
    from shared_prefix_packed_b200 import PackedBatch, _lib

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    name = args.workload
    w = W.WORKLOADS[name]
    P, S = W.group_lengths(name)
    P_all, S_all = P, S
    if args.shard == "groups":
        # strong scaling: one batch, its groups split across the ranks (LPT on pair cost), no data-path collective
        mine = shard_groups(P, S, world)[rank]
        P, S = [P[g] for g in mine], [S[g] for g in mine]
        if not P:
            raise SystemExit(f"rank {rank}: no group to run ({len(P_all)} groups for {world} ranks)")
    inp = W.make_inputs(name, P, S, seed=rank_tensor_seed(name, rank))
    hq, hkv, d = w.num_heads_q, w.num_heads_kv, w.head_dim
    T = W.packed_total(P, S)
    pairs, f_fwd, f_bwd = flops_of(name, P, S)
    stream = torch.cuda.current_stream(dev)

    q, k, v = (inp[x].to(dev) for x in "qkv")
    dout = inp["dout"].to(dev) if w.backward else None
    batch = PackedBatch(P, S, hq, hkv, d, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(hq, T, dtype=torch.float32, device=dev)
    if w.backward:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    n_marks = 5

    def step(marks=None):
        if marks is not None:
            marks[0].record(stream)
        batch.build(stream)
        if marks is not None:
            marks[1].record(stream)
        if w.rope:
            batch.rope(q, k, stream=stream)
        if marks is not None:
            marks[2].record(stream)
        batch.forward(q, k, v, out=o, lse=lse, stream=stream)
        if marks is not None:
            marks[3].record(stream)
        if w.backward:
            batch.backward(q, k, v, o, lse, dout, dq=dq, dk=dk, dv=dv, stream=stream)
        if marks is not None:
            marks[4].record(stream)

    # our kernels per step: metadata (header + 4 stages), RoPE, forward, and the backward's lse/D pass, dK/dV kernel,
    # dQ kernel and split-tile conversion (the workspace memset is a driver memset, not counted)
    launches_per_step = 5 + (1 if w.rope else 0) + 1 + (5 if w.backward else 0)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)                      # nvidia-smi needs a moment before its first sample
    for _ in range(args.warmup):
        step()
    _lib.pp_get_status(stream)

    marks = [[ev() for _ in range(n_marks)] for _ in range(args.steps)]
    t0, t1 = ev(), ev()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for s in range(args.steps):
        step(marks[s])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    _lib.pp_get_status(stream)
    ms = t0.elapsed_time(t1)
    parts = {"build_meta": 0.0, "rope": 0.0, "attn_fwd": 0.0, "attn_bwd": 0.0}
    for m in marks:
        for key, a, b in (("build_meta", 0, 1), ("rope", 1, 2), ("attn_fwd", 2, 3), ("attn_bwd", 3, 4)):
            parts[key] += m[a].elapsed_time(m[b]) / args.steps
    step_ms = [m[0].elapsed_time(m[4]) for m in marks]
    median_ms = max_over_ranks(statistics.median(step_ms), dev, dist)
    ms_per_step = max_over_ranks(ms, dev, dist) / args.steps
    if args.shard == "groups":                     # the whole batch's useful work, once, over the slowest rank
        _, fa, fb = flops_of(name, P_all, S_all)
        job_flops = fa + fb
    else:
        job_flops = (f_fwd + f_bwd) * world

    extras = {}
    if not args.no_extras:
        extras = measure_extras(args, name, P, S, batch, q, k, v, dout, stream, dev)
    value = job_flops / (ms_per_step * 1e-3) / 1e12

    # ---- end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        host = {x: inp[x].pin_memory() for x in (("q", "k", "v", "dout") if w.backward else ("q", "k", "v"))}
        outs = {"dq": torch.empty_like(inp["q"]).pin_memory(), "dk": torch.empty_like(inp["k"]).pin_memory(),
                "dv": torch.empty_like(inp["v"]).pin_memory()} if w.backward else {
            "o": torch.empty_like(inp["q"]).pin_memory(), "lse": torch.empty(hq, T).pin_memory()}
        h2d = sum(t_.numel() * t_.element_size() for t_ in host.values())
        d2h = sum(t_.numel() * t_.element_size() for t_ in outs.values())
        e_steps = max(4, min(args.steps, 10))
        # Two device buffer sets and two copy streams, as a training loop would run it: the uploads of step i+1
        # and the downloads of step i overlap the compute of step i. Every step still copies its inputs in from
        # pinned host memory and its gradients out, inside the timed region; events keep a set's inputs until its
        # step has run and its outputs until they are downloaded.
        in_names = ("q", "k", "v", "dout") if w.backward else ("q", "k", "v")
        out_names = ("dq", "dk", "dv") if w.backward else ("o", "lse")
        set0 = {"q": q, "k": k, "v": v, "dout": dout, "o": o, "lse": lse}
        if w.backward:
            set0.update({"dq": dq, "dk": dk, "dv": dv})
        set1 = {n_: (torch.empty_like(t_) if t_ is not None else None) for n_, t_ in set0.items()}
        sets = [set0, set1]
        hs, ds = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_ready, in_free = [ev(), ev()], [ev(), ev()]
        out_ready, out_free = [ev(), ev()], [ev(), ev()]

        def step_on(B):
            batch.build(stream)
            if w.rope:
                batch.rope(B["q"], B["k"], stream=stream)
            batch.forward(B["q"], B["k"], B["v"], out=B["o"], lse=B["lse"], stream=stream)
            if w.backward:
                batch.backward(B["q"], B["k"], B["v"], B["o"], B["lse"], B["dout"], dq=B["dq"], dk=B["dk"],
                               dv=B["dv"], stream=stream)

        def e2e_run(n, start):
            hs.wait_event(start)
            ds.wait_event(start)
            for st_ in range(n):
                bi = st_ % 2
                B = sets[bi]
                hs.wait_event(in_free[bi])
                with torch.cuda.stream(hs):
                    for n_ in in_names:
                        B[n_].copy_(host[n_], non_blocking=True)
                in_ready[bi].record(hs)
                stream.wait_event(in_ready[bi])
                stream.wait_event(out_free[bi])
                step_on(B)
                in_free[bi].record(stream)
                out_ready[bi].record(stream)
                ds.wait_event(out_ready[bi])
                with torch.cuda.stream(ds):
                    for n_ in out_names:
                        outs[n_].copy_(B[n_], non_blocking=True)
                out_free[bi].record(ds)
            stream.wait_event(out_free[0])
            stream.wait_event(out_free[1])

        for e_ in in_free + out_free:
            e_.record(stream)
        warm = ev()
        warm.record(stream)
        e2e_run(2, warm)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        a, b = ev(), ev()
        a.record(stream)
        e2e_run(e_steps, a)
        b.record(stream)
        torch.cuda.synchronize(dev)
        te = max_over_ranks(a.elapsed_time(b) / e_steps, dev, dist)
        e2e = {"value": round(job_flops / (te * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "ms_per_step": round(te, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks = load_peaks()
    dom = "attn_bwd" if w.backward and parts["attn_bwd"] >= parts["attn_fwd"] else "attn_fwd"
    dom_flops = f_bwd if dom == "attn_bwd" else f_fwd
    achieved = dom_flops / (parts[dom] * 1e-3) / 1e12
    kernels = (["k_bwd_pre", "k_bwd_tc", "k_bwd_dq", "k_bwd_dq_ds", "k_bwd_convert"] if dom == "attn_bwd"
               else ["k_attn_fwd_tc"])
    roofline = {"bound": "tensor", "kernel": f"pp_{dom} ({' + '.join(kernels)})",
                "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16_tflops"], 4), "traffic": recorded_traffic(kernels, name),
                "peak_source": peaks["source"] + " bf16_tflops (burst)",
                "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4)
                if peaks.get("bf16_tflops_sustained") else None,
                "flops_per_launch": dom_flops, "ms_per_launch": round(parts[dom], 4)}
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(name, P, S, seconds=args.cpu_seconds)
    line = {
        "metric": "packed-prefix attn fwd+bwd useful TFLOP/s", "value": round(value, 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "strong" if args.shard == "groups" else "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16"
        else "fp32", "data": "synthetic",
        "config": {"workload": f"{name}: {w.description}", "T": T, "groups": len(P), "allowed_pairs_per_head": pairs,
                   "unpacked_pairs_per_head": unpacked_pairs(P, S), "useful_gflop_per_rank": (f_fwd + f_bwd) / 1e9,
                   "l2": f"inputs larger than L2 ({(q.numel() + k.numel() + v.numel()) * 2 / 2**20:.0f} MiB of Q/K/V "
                         f"per rank vs 126 MiB), no flush",
                   "parallelism": (f"one batch's groups split across {world} ranks (LPT on pair cost)"
                                   if args.shard == "groups" else f"weak-scaled replicas x{world}")},
        "frac_of_peak": round(value / world / peaks["bf16_tflops"], 4),
        "frac_of_peak_sustained": round(value / world / peaks["bf16_tflops_sustained"], 4)
        if peaks.get("bf16_tflops_sustained") else None,
        "frac_of_datasheet": round(value / world / DATASHEET_BF16_TFLOPS, 4),
        "datasheet": {"bf16_dense_tflops": DATASHEET_BF16_TFLOPS, "source": DATASHEET_SOURCE},
        "step_ms_median": round(median_ms, 4), "step_ms_mean": round(ms_per_step, 4),
        "ms_per_call": {k_: round(v_, 4) for k_, v_ in parts.items()},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    line.update(extras)
    print(json.dumps(line), flush=True)


def _timed(fn, reps, stream, flush=None):
    """Median device time (ms) of fn() over reps calls, each timed alone with CUDA events on `stream`; flush() (an
    L2-sized write) runs before every call, outside the timed span."""
    import torch
    out = []
    for _ in range(reps):
        if flush is not None:
            flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        out.append(a.elapsed_time(b))
    return statistics.median(out)


def measure_extras(args, name, P, S, batch, q, k, v, dout, stream, dev, reps=20):
    """Measurements beside the headline step (same rank, after its timed region):
      * pp_rope and pp_build_meta alone, each after an L2 flush (a 256 MiB write), as GB/s of their algorithmic
        bytes: RoPE reads and writes Q and K once and reads the position ids; the builder reads the descriptors and
        segment bounds and writes the position ids, the two per-token tables and the tile lists;
      * the unpacked comparison: the same four calls on the same preference samples laid out without packing (every
        response its own sequence P || S_i), with its allowed pairs, K/V bytes and step time."""
    import torch
    from shared_prefix_packed_b200 import PackedBatch, _lib
    w = W.WORKLOADS[name]
    hq, hkv, d = w.num_heads_q, w.num_heads_kv, w.head_dim
    T = W.packed_total(P, S)
    flush_buf = torch.empty(64 * 2 ** 20, dtype=torch.float32, device=dev)
    flush = lambda: flush_buf.fill_(1.0)  # noqa: E731
    peaks = load_peaks()
    res = {}
    hdr = batch.meta[:64].view(torch.int32).cpu().tolist()
    n_qt, n_kt, n_bw = hdr[6], hdr[7], hdr[8]
    G, nseg = len(P), sum(1 + len(ss) for ss in S)
    meta_bytes = 8 * G + 4 * (nseg + 1) + 4 * T + 8 * T + 2 * 48 * n_qt + 32 * n_kt + 32 * n_bw
    ms_meta = _timed(lambda: batch.build(stream), reps, stream, flush)
    res["meta"] = {"ms": round(ms_meta, 4), "bytes": meta_bytes, "gbs": round(meta_bytes / (ms_meta * 1e-3) / 1e9, 1),
                   "launches": 5, "note": "five launches of a few us each: launch-latency bound at this size"}
    if w.rope:
        rope_bytes = T * (hq + hkv) * d * 2 * 2 + 4 * T
        ms_rope = _timed(lambda: batch.rope(q, k, stream=stream), reps, stream, flush)
        gbs = rope_bytes / (ms_rope * 1e-3) / 1e9
        res["rope"] = {"ms": round(ms_rope, 4), "bytes": rope_bytes, "gbs": round(gbs, 1),
                       "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4), "l2": "flushed (256 MiB write) before each call"}
    # unpacked comparison
    Pu, Su = unpacked_layout(P, S)
    Tu = W.packed_total(Pu, Su)
    inp = W.make_inputs(name, Pu, Su, seed=w.tensor_seed + 17)
    qu, ku, vu = (inp[x].to(dev) for x in "qkv")
    bu = PackedBatch(Pu, Su, hq, hkv, d, device=dev)
    ou = torch.empty_like(qu)
    lu = torch.empty(hq, Tu, dtype=torch.float32, device=dev)
    if w.backward:
        du = inp["dout"].to(dev)
        gq, gk, gv = torch.empty_like(qu), torch.empty_like(ku), torch.empty_like(vu)

    def ustep():
        bu.build(stream)
        if w.rope:
            bu.rope(qu, ku, stream=stream)
        bu.forward(qu, ku, vu, out=ou, lse=lu, stream=stream)
        if w.backward:
            bu.backward(qu, ku, vu, ou, lu, du, dq=gq, dk=gk, dv=gv, stream=stream)

    o_ = torch.empty_like(q)
    l_ = torch.empty(hq, T, dtype=torch.float32, device=dev)
    if w.backward:
        g_ = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))

    def pstep():
        batch.build(stream)
        if w.rope:
            batch.rope(q, k, stream=stream)
        batch.forward(q, k, v, out=o_, lse=l_, stream=stream)
        if w.backward:
            batch.backward(q, k, v, o_, l_, dout, dq=g_[0], dk=g_[1], dv=g_[2], stream=stream)

    for _ in range(3):
        ustep()
    _lib.pp_get_status(stream)
    ms_u = _timed(ustep, reps, stream)
    ms_p = _timed(pstep, reps, stream)
    pairs_p, pairs_u = pair_count(P, S), pair_count(Pu, Su)
    kv_p, kv_u = 2 * T * hkv * d * 2, 2 * Tu * hkv * d * 2
    fl = (4 + (10 if w.backward else 0)) * d * hq
    res["unpacked"] = {
        "layout": "every response its own sequence P || S_i (same samples, no packing)",
        "T": Tu, "allowed_pairs_per_head": pairs_u, "kv_bytes": kv_u, "ms_per_step": round(ms_u, 4),
        "tflops_on_its_own_pairs": round(fl * pairs_u / (ms_u * 1e-3) / 1e12, 1),
        "packed_ms_per_step_same_timing": round(ms_p, 4),
        "speedup_packed_over_unpacked": round(ms_u / ms_p, 3),
        "pairs_saved": round(1 - pairs_p / pairs_u, 4), "kv_bytes_saved": round(1 - kv_p / kv_u, 4),
        "timing": f"median of {reps} single steps each (CUDA events), both layouts timed the same way"}
    del qu, ku, vu, ou, lu, bu
    return res


# ---------------------------------------------------------------------------------------------------- CPU oracle
def cpu_baseline(name, P, S, seconds=15.0, steps=1):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload: whole groups, fwd (+bwd)."""
    import oracle
    w = W.WORKLOADS[name]
    inp = W.make_inputs(name, P, S)
    lay = oracle.layout_of(P, S)
    hq, hkv = w.num_heads_q, w.num_heads_kv
    r = hq // hkv
    # take one kv head (and its r q heads) of as many groups as fit roughly in the budget, smallest first
    order = sorted(range(len(P)), key=lambda g: int(lay.group_len[g]))
    chosen, flops, t_used = [], 0, 0.0
    t_start = time.perf_counter()
    for g in order:
        if chosen and time.perf_counter() - t_start > seconds:
            break
        gp = pair_count([P[g]], [S[g]])
        t0 = time.perf_counter()
        oracle.attention_forward(inp["q"], inp["k"], inp["v"], P, S, heads=list(range(r)), groups=[g])
        if w.backward:
            oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["dout"], P, S, groups=[g], kv_heads=[0])
        t_used += time.perf_counter() - t0
        flops += (4 + (10 if w.backward else 0)) * w.head_dim * gp * r
        chosen.append(g)
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # pragma: no cover
        cores = 1
    return {"value": round(flops / t_used / 1e12, 6), "unit": "TFLOP/s", "cores": int(cores), "kind": "oracle",
            "sample": f"{len(chosen)} whole group(s) of {len(P)}, kv head 0 with its {r} q heads, "
                      f"fwd{'+bwd' if w.backward else ''}, fp64 numpy ({flops / 1e9:.1f} useful GFLOP in "
                      f"{t_used:.1f} s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = args.workload
    P, S = W.group_lengths(name)
    per = []
    info = None
    for _ in range(args.warmup + args.steps):
        info = cpu_baseline(name, P, S, seconds=args.cpu_seconds / max(1, args.steps))
        per.append(info)
    vals = [x["value"] for x in per[args.warmup:]]
    value = statistics.median(vals)
    w = W.WORKLOADS[name]
    line = {"impl": "reference", "metric": "packed-prefix attn fwd+bwd useful TFLOP/s", "value": value,
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{name}: {w.description}", "T": W.packed_total(P, S)},
            "cpu_baseline": {"kind": "oracle", "cores": info["cores"], "sample": info["sample"], "value": value},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_batcher(args):
    """The host batch planner (pp_plan_batches) and the work model behind "packing combines with batch sorting".

    Throughput: plans per second over one million synthetic groups (host code, host clock). Work model, on 20,000
    synthetic groups with the dpo length distribution (P ~ U[512, 2048], two responses ~ U[128, 1024]): the tokens
    and causal attention pairs a padded implementation processes with 8 groups per batch, for
      baseline   one sequence per (prompt, response), dataset order, padded to the batch's longest;
      sorted     the same with the groups sorted by length first;
      packed     one sequence per group (prompt once, then its responses), dataset order, padded;
      packed+sorted,
    and the pad-free packed form these kernels run (capacity batches from pp_plan_batches, no padding, only the
    allowed pairs of the packed mask)."""
    from shared_prefix_packed_b200 import pp_plan_batches

    rng = np.random.default_rng(5001)
    n_big = 1_000_000
    toks = rng.integers(512, 2049, size=n_big) + rng.integers(128, 1025, size=(n_big, 2)).sum(axis=1)
    pp_plan_batches(toks[:1000], 65536, True)
    t0 = time.perf_counter()
    for _ in range(3):
        pp_plan_batches(toks, 65536, True)
    plan_s = (time.perf_counter() - t0) / 3

    n = 20000
    P = rng.integers(512, 2049, size=n)
    Sr = rng.integers(128, 1025, size=(n, 2))
    B = 8                                                     # groups per padded batch

    def padded(lengths_per_group, order):
        tok = pairs = 0
        for b0 in range(0, n, B):
            seqs = [L for g in order[b0:b0 + B] for L in lengths_per_group[g]]
            mx = max(seqs)
            tok += len(seqs) * mx
            pairs += len(seqs) * mx * (mx + 1) // 2
        return tok, pairs

    unpacked = [[int(P[g] + Sr[g, 0]), int(P[g] + Sr[g, 1])] for g in range(n)]
    packed = [[int(P[g] + Sr[g].sum())] for g in range(n)]
    ident = list(range(n))
    by_unp = sorted(ident, key=lambda g: -max(unpacked[g]))
    by_pk = sorted(ident, key=lambda g: -packed[g][0])
    rows = {"baseline": padded(unpacked, ident), "sorted": padded(unpacked, by_unp),
            "packed": padded(packed, ident), "packed+sorted": padded(packed, by_pk)}
    useful_tok = int(P.sum() + Sr.sum())
    useful_pairs = int(sum(p * (p + 1) // 2 + sum(s * p + s * (s + 1) // 2 for s in Sr[g]) for g, p in enumerate(P)))
    order, batch, nb = pp_plan_batches([packed[g][0] for g in range(n)], 65536, True)
    rows["pad-free packed (these kernels)"] = (useful_tok, useful_pairs)
    base_tok, base_pairs = rows["baseline"]
    model = {k: {"tokens": v[0], "attention_pairs": v[1], "token_speedup": round(base_tok / v[0], 3),
                 "attention_speedup": round(base_pairs / v[1], 3)} for k, v in rows.items()}
    print(json.dumps({
        "metric": "host batch planning groups/s", "value": round(n_big / plan_s, 1), "unit": "groups/s",
        "n_gpus": 0, "steps": 3, "warmup": 1, "ms_per_step": round(plan_s * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
        "config": {"workload": f"{n_big} groups of the dpo length mix, capacity 65,536 tokens, sorted",
                   "model_groups": n, "model_batch_groups": B, "pad_free_batches": nb},
        "modeled_work": model}))


def run_decode(args):
    """One decoding step of every response over the workload's layout as a group-contiguous KV cache
    (pp_decode_attn): one query per response (its newest token), 32/8 heads, d = 128. HBM-bound; the algorithmic
    bytes are the cache read once (a prefix serves all responses of its group) plus the queries and outputs."""
    import torch
    from shared_prefix_packed_b200 import PackedBatch, _lib

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    name = args.workload
    P, S = W.group_lengths(name)
    w = W.WORKLOADS[name]
    hq, hkv, d = w.num_heads_q, w.num_heads_kv, w.head_dim
    T = W.packed_total(P, S)
    n_resp = sum(len(ss) for ss in S)
    gen = torch.Generator(device=dev)
    gen.manual_seed(3001)
    k = torch.randn(T, hkv, d, generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn(T, hkv, d, generator=gen, device=dev).to(torch.bfloat16)
    q = torch.randn(n_resp, hq, d, generator=gen, device=dev).to(torch.bfloat16)
    batch = PackedBatch(P, S, hq, hkv, d, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(hq, n_resp, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    nbytes = 2 * T * hkv * d * 2 + 2 * n_resp * hq * d * 2 + n_resp * hq * 4
    unpacked = sum((p + s) * hkv * d * 2 * 2 for p, ss in zip(P, S) for s in ss)
    for _ in range(args.warmup):
        batch.decode(q, k, v, out=o, lse=lse, stream=stream)
    _lib.pp_get_status(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for _ in range(args.steps):
        batch.decode(q, k, v, out=o, lse=lse, stream=stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / args.steps
    gbs = nbytes / (ms * 1e-3) / 1e9
    peaks = load_peaks()
    print(json.dumps({
        "metric": "decode step over a group-contiguous KV cache GB/s", "value": round(gbs, 1), "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{name} layout as the KV cache: T={T}, {n_resp} responses, {hq}/{hkv} heads, d={d}",
                   "cache_bytes_read_once": 2 * T * hkv * d * 2,
                   "cache_bytes_if_unpacked": unpacked,
                   "l2": f"K/V cache {2 * T * hkv * d * 2 / 2**20:.0f} MiB, larger than L2, no flush"},
        "roofline": {"bound": "hbm", "kernel": "k_dec_plan + k_dec_chunk + k_dec_combine", "achieved": round(gbs, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "traffic": None, "peak_source": peaks["source"] + " hbm_gbs", "bytes_per_launch": nbytes},
        "gpu_launches": 3 * args.steps}))


def run_pack(args):
    """Device-side packing of an ungrouped micro-batch (pp_pack_batch, the step before the path) on the workload's
    groups: every sample carries its group's prompt (left-padded to the longest prompt) and its own response
    (right-padded), samples of a group share a uid. Tiny and launch-bound; bytes = the masks and ids read plus the
    packed ids written."""
    import torch
    from shared_prefix_packed_b200 import _lib

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    name = args.workload
    P, S = W.group_lengths(name)
    rng = np.random.default_rng(4001)
    samples = [(g, p, s) for g, (p, ss) in enumerate(zip(P, S)) for s in ss]
    bs = len(samples)
    Lp, Lr = max(P), max(s for _, _, s in samples)
    prompts = np.zeros((bs, Lp), np.int32)
    pm = np.zeros((bs, Lp), np.uint8)
    responses = np.zeros((bs, Lr), np.int32)
    rm = np.zeros((bs, Lr), np.uint8)
    group_prompt = [rng.integers(0, W.LOGPROB_VOCAB, size=p) for p in P]
    for i, (g, p, s) in enumerate(samples):
        prompts[i, Lp - p:] = group_prompt[g]
        pm[i, Lp - p:] = 1
        responses[i, :s] = rng.integers(0, W.LOGPROB_VOCAB, size=s)
        rm[i, :s] = 1
    uids = np.array([g for g, _, _ in samples], np.int64)
    t = lambda x: torch.from_numpy(x).to(dev)
    d_p, d_pm, d_r, d_rm, d_u = t(prompts), t(pm), t(responses), t(rm), t(uids)
    packed = torch.empty(bs * (Lp + Lr), dtype=torch.int32, device=dev)
    groups = torch.empty(bs, 2, dtype=torch.int32, device=dev)
    cu = torch.empty(2 * bs + 1, dtype=torch.int32, device=dev)
    off = torch.empty(bs, 2, dtype=torch.int32, device=dev)
    counts = torch.empty(3, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    call = lambda: _lib.pp_pack_batch(d_p, d_pm, d_r, d_rm, d_u, packed, groups, cu, off, counts, stream)
    for _ in range(args.warmup):
        call()
    _lib.pp_get_status(stream)
    T = int(counts[2])
    nbytes = bs * (Lp + Lr) * 5 + bs * 8 + T * 4 + (2 * bs + 1) * 4
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for _ in range(args.steps):
        call()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / args.steps
    gbs = nbytes / (ms * 1e-3) / 1e9
    peaks = load_peaks()
    print(json.dumps({
        "metric": "micro-batch packing GB/s", "value": round(gbs, 2), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int32", "data": "synthetic",
        "config": {"workload": f"{name} groups as an ungrouped micro-batch: bs={bs}, Lp={Lp}, Lr={Lr}, T={T}",
                   "note": "three launches per call; launch-latency bound at this size"},
        "roofline": {"bound": "hbm", "kernel": "k_pack_count + k_pack_layout + k_pack_gather",
                     "achieved": round(gbs, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / peaks["hbm_gbs"], 5), "traffic": None,
                     "peak_source": peaks["source"] + " hbm_gbs", "bytes_per_launch": nbytes},
        "gpu_launches": 3 * args.steps}))


def run_logprobs(args):
    """The response log-probability read-out on its own (the row after attention): one pp_response_logprobs call
    per step over the packed logits of the workload's layout at a 151,936-entry vocabulary. HBM-bound: the
    algorithmic bytes are one logits row per scored token, plus the token ids and the output."""
    import torch
    from shared_prefix_packed_b200 import PackedBatch, _lib

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    name = args.workload
    P, S = W.group_lengths(name)
    T = W.packed_total(P, S)
    V = args.vocab
    gen = torch.Generator(device=dev)
    gen.manual_seed(2001)
    logits = (torch.randn(T, V, generator=gen, device=dev, dtype=torch.float32) * W.LOGPROB_LOGIT_STD).to(
        torch.bfloat16)
    ids = torch.randint(0, V, (T,), generator=gen, device=dev, dtype=torch.int32)
    w = W.WORKLOADS[name]
    batch = PackedBatch(P, S, w.num_heads_q, w.num_heads_kv, w.head_dim, device=dev)
    out = torch.empty(T, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # scored rows: every response token, except the first token of each non-empty response of a group with no prefix
    scored = sum(sum(ss) - (sum(1 for x in ss if x > 0) if p == 0 else 0) for p, ss in zip(P, S))
    nbytes = scored * V * 2 + T * 4 * 2
    for _ in range(args.warmup):
        batch.response_logprobs(logits, ids, 0.9, out=out, stream=stream)
    _lib.pp_get_status(stream)
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for _ in range(args.steps):
        batch.response_logprobs(logits, ids, 0.9, out=out, stream=stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    _lib.pp_get_status(stream)
    ms = t0.elapsed_time(t1) / args.steps
    gbs = nbytes / (ms * 1e-3) / 1e9
    peaks = load_peaks()
    print(json.dumps({
        "metric": "response log-prob read-out GB/s", "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{name} layout, T={T}, scored rows={scored}, vocab={V}, bf16 logits ~ N(0, 4^2)",
                   "l2": f"logits {T * V * 2 / 2**30:.1f} GiB, larger than L2, no flush"},
        "roofline": {"bound": "hbm", "kernel": "k_response_logprobs", "achieved": round(gbs, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "traffic": recorded_traffic(["k_response_logprobs"], f"{name}-layout-vocab{V}"),
                     "peak_source": peaks["source"] + " hbm_gbs", "bytes_per_launch": nbytes},
        "gpu_launches": args.steps, "clocks": clocks}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "groups"],
                    help="N>1: every rank its own batch (weak scaling, default) or one batch's groups split across the "
                         "ranks by LPT on pair cost (strong scaling)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the rope/meta GB/s and the unpacked comparison measured after the timed region")
    ap.add_argument("--vocab", type=int, default=W.LOGPROB_VOCAB, help="vocabulary of the --logprobs read-out")
    ap.add_argument("--batcher", action="store_true",
                    help="host batch planner throughput and the modeled work of packing with batch sorting")
    ap.add_argument("--decode", action="store_true",
                    help="time one decoding step over the workload's layout as a KV cache (pp_decode_attn)")
    ap.add_argument("--pack", action="store_true",
                    help="time device-side packing of an ungrouped micro-batch (pp_pack_batch)")
    ap.add_argument("--logprobs", action="store_true",
                    help="time the response log-prob read-out (pp_response_logprobs) instead of the attention step")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.batcher:
        run_batcher(args)
    elif args.decode:
        run_decode(args)
    elif args.pack:
        run_pack(args)
    elif args.logprobs:
        run_logprobs(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
