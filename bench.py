#!/usr/bin/env python
"""Benchmark of the B200 HSA forward path (landmarks -> top-k selection ->
chunk attention + fusion), through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

One step is one pass of the whole path over one prefill sequence of the
prefill_bf16 workload (B1, T 65536, H32/Hkv8, d128, S64, k16, bf16).  Ranks
under torchrun each run their own sequence (weak scaling; no data-path
collective).  The timed region is bracketed by a barrier and a device
synchronise, and timed with CUDA events on the launching stream.  The reported
time is the maximum over ranks.  The inputs (Q 512 MiB, K and V 128 MiB each)
are larger than L2, so no flush is needed between prefill steps.  The decode
lines (decode_1m: batch 8, 1M cached tokens; decode_16m: batch 1, 16M cached
tokens) flush L2 before every step.

--impl reference times the CPU oracle instead (the task has no other
reference implementation), on a bounded sample of the same workload.
Rank 0 alone runs it.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "HSA prefill tokens/s & decode µs/token at 1M ctx; % of HBM / tensor roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


# --------------------------------------------------------------------------- distributed plumbing

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.gpu = str(device)
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.out.flush()
        self.out.seek(0)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.read().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.out.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- algorithmic work

def ncand_rows(p) -> np.ndarray:
    t = np.arange(p.Tq, dtype=np.int64)
    return np.minimum((p.q_pos0 + t) // p.S, p.C)


def work_counts(p, keff_sum: int) -> dict:
    """Algorithmic work of one forward call (what the method must do: causal
    candidate chunks only, k_eff chunks of S keys per query head)."""
    es = 2 if p.dtype == "bf16" else 4
    lm_bytes = (p.B * p.Tkv * p.Hkv * p.d + p.d * p.d + p.B * p.Hkv * p.C * p.d) * es
    sel_flops = 2.0 * p.d * p.H * float(ncand_rows(p).sum()) * p.B
    att_flops = 4.0 * p.S * p.d * p.G * float(keff_sum)
    att_bytes = (2 * p.B * p.Tq * p.H * p.d) * es + 2 * p.B * p.Tkv * p.Hkv * p.d * es
    return {"landmarks_bytes": lm_bytes, "select_flops": sel_flops, "attend_flops": att_flops,
            "attend_bytes": att_bytes}


# --------------------------------------------------------------------------- our arm

class PrefillSetup:
    """Inputs, outputs and the three stage calls (landmarks, select, attend) of
    one prefill workload, each a direct call of the C ABI on one stream."""

    def __init__(self, name, seed, dev):
        import landmark_guided_chunk_b200 as hsa
        from landmark_guided_chunk_b200.inputs import make_inputs, workload

        self.hsa = hsa
        self.dev = dev
        self.p = p = workload(name)
        self.inp = make_inputs(p, seed=seed, device=dev)
        self.Q, self.K, self.V, self.W = (self.inp[x] for x in ("Q", "K", "V", "W_L"))
        self.prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau,
                                     torch.bfloat16 if p.dtype == "bf16" else torch.float32)
        self.plan = hsa.plan(self.prob)
        self.ws = hsa.alloc_workspace(self.prob, dev)
        self.L = torch.empty(p.B, p.Hkv, p.C, p.d, dtype=self.Q.dtype, device=dev)
        self.O = torch.empty_like(self.Q)
        km = hsa.kmax_of(p.k, p.tau)
        self.idx = torch.empty(p.B, p.Tq, p.Hkv, km, dtype=torch.int32, device=dev)
        self.score = torch.empty(p.B, p.Tq, p.Hkv, km, dtype=torch.float32, device=dev)
        self.keff = torch.empty(p.B, p.Tq, p.Hkv, dtype=torch.int32, device=dev)
        self.st = torch.cuda.current_stream(dev)
        lib, P, sp, prob = hsa._native.lib(), hsa._p, self.st.cuda_stream, self.prob
        Q, K, V, W, L, O = self.Q, self.K, self.V, self.W, self.L, self.O
        idx, score, keff, ws = self.idx, self.score, self.keff, self.ws

        def stage_landmarks():
            hsa._native.check(lib.hsa_landmarks(ctypes.byref(prob), P(K), P(W), P(L), sp), "hsa_landmarks")

        def stage_select():
            hsa._native.check(lib.hsa_select(ctypes.byref(prob), P(Q), P(L), P(idx), P(score), P(keff), P(ws),
                                             ws.numel(), sp), "hsa_select")

        def stage_attend():
            hsa._native.check(lib.hsa_attend(ctypes.byref(prob), P(Q), P(K), P(V), P(idx), P(score), P(keff),
                                             P(O), P(ws), ws.numel(), sp), "hsa_attend")

        self.stages = [("landmarks", stage_landmarks), ("select", stage_select), ("attend", stage_attend)]

    def time_stages(self, steps, warmup, world, clocks=None):
        """Warm-up, then `steps` forwards back to back, each stage bracketed by
        CUDA events on the launching stream.  Returns (ms per forward, max over
        ranks; mean ms of each stage; keff sum; clock record)."""
        for _ in range(warmup):
            for _, f in self.stages:
                f()
        torch.cuda.synchronize(self.dev)
        keff_sum = int(self.keff.sum().item())
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize(self.dev)
        if clocks is not None:
            clocks.start()
        for s in range(steps):
            ev[s][0].record(self.st)
            for i, (_, f) in enumerate(self.stages):
                f()
                ev[s][i + 1].record(self.st)
        torch.cuda.synchronize(self.dev)
        clk = clocks.stop() if clocks is not None else None
        barrier(world)
        total_ms = sum(e[0].elapsed_time(e[3]) for e in ev)
        stage_ms = {name: sum(e[i].elapsed_time(e[i + 1]) for e in ev) / steps
                    for i, (name, _) in enumerate(self.stages)}
        return max_over_ranks(total_ms / steps, world), stage_ms, keff_sum, clk

    def roofline(self, stage_ms, keff_sum, pk):
        """Each stage's achieved rate against the measured peaks, and the
        dominant stage's roofline object.  The stages are timed inside a
        forward of a few ms, so the burst bf16 peak applies; the fraction of
        the sustained peak is given beside it."""
        p, work = self.p, work_counts(self.p, keff_sum)
        stage_rf = {
            "landmarks": {"bound": "hbm", "work": work["landmarks_bytes"], "unit": "GB/s", "peak": pk["hbm_gbs"]},
            "select": {"bound": "tensor", "work": work["select_flops"], "unit": "TFLOP/s", "peak": pk["bf16_tflops"]},
            "attend": {"bound": "tensor", "work": work["attend_flops"], "unit": "TFLOP/s", "peak": pk["bf16_tflops"]},
        }
        stages_out = {}
        for name, rf in stage_rf.items():
            ms = stage_ms[name]
            scale = 1e-9 if rf["unit"] == "GB/s" else 1e-12
            ach = rf["work"] * scale / (ms * 1e-3)
            stages_out[name] = {"ms": round(ms, 4), "path": self.plan[name][0], "kernels": self.plan[name][1],
                                "achieved": round(ach, 2), "unit": rf["unit"], "bound": rf["bound"],
                                "frac": round(ach / rf["peak"], 4)}
            if rf["unit"] == "TFLOP/s":
                stages_out[name]["frac_of_sustained"] = round(ach / pk["bf16_tflops_sustained"], 4)
        dom = max(stage_ms, key=stage_ms.get)
        traffic = dram_traffic(f"{dom}:{p.name}", self.plan[dom][0])
        roof = {"bound": stage_rf[dom]["bound"], "kernel": f"hsa_{dom} ({self.plan[dom][0]})",
                "achieved": stages_out[dom]["achieved"], "peak": stage_rf[dom]["peak"],
                "unit": stage_rf[dom]["unit"], "frac": stages_out[dom]["frac"], "traffic": traffic,
                "peak_source": f"{pk['source']} ({'burst bf16' if stage_rf[dom]['unit'] == 'TFLOP/s' else 'HBM copy'})"}
        return stages_out, roof


def run_router(args, world, rank, local, pk):
    """The gap-router prefill workload (router_bf16: B1, T 131072, S 128, k 8
    doubled to 16 where the normalised top-k gap is below tau = 0.02): forward
    time per stage, tokens/s, the mean k_eff and the measured fraction of
    selection rows the router doubled."""
    dev = torch.device("cuda", local)
    ps = PrefillSetup("router_bf16", args.seed + rank, dev)
    p = ps.p
    steps = max(1, min(args.steps, 10))
    ms, stage_ms, keff_sum, _ = ps.time_stages(steps, args.warmup, world)
    stages_out, roof = ps.roofline(stage_ms, keff_sum, pk)
    nc = torch.as_tensor(ncand_rows(p), device=dev).view(1, -1, 1)
    eligible = (nc > p.k).expand_as(ps.keff)
    doubled = (ps.keff > p.k) & eligible
    frac = float(doubled.sum().item()) / max(1, int(eligible.sum().item()))
    out = {"workload": f"{p.name}: B{p.B} T{p.Tq} H{p.H} Hkv{p.Hkv} d{p.d} S{p.S} k{p.k}->{2 * p.k} tau{p.tau}",
           "ms_per_forward": round(ms, 4), "steps": steps, "tokens_per_s": round(p.B * p.Tq * world / (ms * 1e-3), 1),
           "keff_mean": round(keff_sum / (p.B * p.Tq * p.Hkv), 3), "doubled_fraction": round(frac, 4),
           "stages": stages_out, "roofline": roof,
           "gpu_launches": steps * sum(ps.plan[x][1] for x in ("landmarks", "select", "attend"))}
    del ps
    torch.cuda.empty_cache()
    return out


def run_prefill_line(args, world, rank, local, pk, name):
    """Another prefill workload (prefill_bf16_d64: the prefill_bf16 shapes at head
    dim 64) through the same forward: time per stage, tokens/s, roofline."""
    dev = torch.device("cuda", local)
    ps = PrefillSetup(name, args.seed + rank, dev)
    p = ps.p
    steps = max(1, min(args.steps, 10))
    ms, stage_ms, keff_sum, _ = ps.time_stages(steps, args.warmup, world)
    stages_out, roof = ps.roofline(stage_ms, keff_sum, pk)
    out = {"workload": f"{p.name}: B{p.B} T{p.Tq} H{p.H} Hkv{p.Hkv} d{p.d} S{p.S} k{p.k}",
           "ms_per_forward": round(ms, 4), "steps": steps, "tokens_per_s": round(p.B * p.Tq * world / (ms * 1e-3), 1),
           "stages": stages_out, "roofline": roof,
           "gpu_launches": steps * sum(ps.plan[x][1] for x in ("landmarks", "select", "attend"))}
    del ps
    torch.cuda.empty_cache()
    return out


def run_variants(args, world, rank, local, pk):
    """The two selection variants on the prefill_bf16 shapes, each stage timed
    with CUDA events over back-to-back forwards: Quest block scoring
    (summaries -> Quest selection -> attention) and the landmark refiner
    (refined landmarks -> selection -> attention)."""
    import landmark_guided_chunk_b200 as hsa

    dev = torch.device("cuda", local)
    ps = PrefillSetup(args.workload, args.seed + rank, dev)
    p, Q, K, V, W = ps.p, ps.Q, ps.K, ps.V, ps.W
    lib, P, sp = hsa._native.lib(), hsa._p, ps.st.cuda_stream
    g = torch.Generator(device=dev).manual_seed(args.seed + 7)
    Wq, Wk, Wv = ((torch.randn(p.d, p.d, device=dev, generator=g) / math.sqrt(p.d)).to(Q.dtype) for _ in range(3))
    steps = max(1, min(args.steps, 10))
    out = {}
    es = 2 if p.dtype == "bf16" else 4
    k_bytes = p.B * p.Tkv * p.Hkv * p.d * es

    def timed(stages):
        for _ in range(args.warmup):
            for _, f in stages:
                f()
        torch.cuda.synchronize(dev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(steps)]
        barrier(world)
        for s in range(steps):
            ev[s][0].record(ps.st)
            for i, (_, f) in enumerate(stages):
                f()
                ev[s][i + 1].record(ps.st)
        torch.cuda.synchronize(dev)
        barrier(world)
        ms = {name: sum(e[i].elapsed_time(e[i + 1]) for e in ev) / steps for i, (name, _) in enumerate(stages)}
        return ms, max_over_ranks(sum(ms.values()), world)

    # Quest block scoring
    qprob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, Q.dtype,
                             hsa._native.HSA_FLAG_QUEST)
    qplan = hsa.plan(qprob)
    qws = hsa.alloc_workspace(qprob, dev)
    Lq = torch.empty(p.B, p.Hkv, p.C, 2 * p.d, dtype=Q.dtype, device=dev)
    idx, score, keff, O = ps.idx, ps.score, ps.keff, ps.O
    stages = [
        ("summaries", lambda: hsa._native.check(lib.hsa_landmarks(ctypes.byref(qprob), P(K), None, P(Lq), sp),
                                                "hsa_landmarks")),
        ("select", lambda: hsa._native.check(lib.hsa_select(ctypes.byref(qprob), P(Q), P(Lq), P(idx), P(score),
                                                            P(keff), P(qws), qws.numel(), sp), "hsa_select")),
        ("attend", lambda: hsa._native.check(lib.hsa_attend(ctypes.byref(qprob), P(Q), P(K), P(V), P(idx),
                                                            P(score), P(keff), P(O), P(qws), qws.numel(), sp),
                                             "hsa_attend")),
    ]
    ms, total = timed(stages)
    keff_sum = int(keff.sum().item())
    work = work_counts(p, keff_sum)
    # the selection kernels contract [P | N] (hi and lo parts) with [Mx | Mn]: 4d per (token, kv head, candidate)
    sel_flops = 2.0 * 4 * p.d * p.Hkv * float(ncand_rows(p).sum()) * p.B
    sum_bytes = k_bytes + p.B * p.Hkv * p.C * 2 * p.d * es
    out["quest"] = {
        "ms_per_forward": round(total, 4), "tokens_per_s": round(p.B * p.Tq * world / (total * 1e-3), 1),
        "keff_mean": round(keff_sum / (p.B * p.Tq * p.Hkv), 3), "plan": {k2: (list(v) if isinstance(v, tuple) else v) for k2, v in qplan.items()},
        "stages": {
            "summaries": {"ms": round(ms["summaries"], 4), "bound": "hbm", "unit": "GB/s",
                          "achieved": round(sum_bytes / (ms["summaries"] * 1e-3) / 1e9, 1),
                          "frac": round(sum_bytes / (ms["summaries"] * 1e-3) / 1e9 / pk["hbm_gbs"], 4)},
            "select": {"ms": round(ms["select"], 4), "bound": "tensor", "unit": "TFLOP/s",
                       "achieved": round(sel_flops / (ms["select"] * 1e-3) / 1e12, 2),
                       "frac": round(sel_flops / (ms["select"] * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
                       "note": "query transform + tcgen05 scoring of the width-4d contraction with fused top-k"},
            "attend": {"ms": round(ms["attend"], 4), "bound": "tensor", "unit": "TFLOP/s",
                       "achieved": round(work["attend_flops"] / (ms["attend"] * 1e-3) / 1e12, 2),
                       "frac": round(work["attend_flops"] / (ms["attend"] * 1e-3) / 1e12 / pk["bf16_tflops"], 4)}},
        "gpu_launches": steps * sum(qplan[x][1] for x in ("landmarks", "select", "attend"))}
    del qws, Lq

    # landmark refiner
    L = ps.L

    def refine():
        hsa._native.check(lib.hsa_landmarks_refined(ctypes.byref(ps.prob), P(K), P(W), P(Wq), P(Wk), P(Wv), P(L), sp),
                          "hsa_landmarks_refined")

    stages = [("refined_landmarks", refine)] + ps.stages[1:]
    ms, total = timed(stages)
    keff_sum = int(keff.sum().item())
    lm_bytes = k_bytes + p.B * p.Hkv * p.C * p.d * es + 4 * p.d * p.d * es
    out["refine"] = {
        "ms_per_forward": round(total, 4), "tokens_per_s": round(p.B * p.Tq * world / (total * 1e-3), 1),
        "keff_mean": round(keff_sum / (p.B * p.Tq * p.Hkv), 3),
        "stages": {"refined_landmarks": {"ms": round(ms["refined_landmarks"], 4), "bound": "hbm", "unit": "GB/s",
                                         "achieved": round(lm_bytes / (ms["refined_landmarks"] * 1e-3) / 1e9, 1),
                                         "frac": round(lm_bytes / (ms["refined_landmarks"] * 1e-3) / 1e9
                                                       / pk["hbm_gbs"], 4)},
                   "select": {"ms": round(ms["select"], 4)}, "attend": {"ms": round(ms["attend"], 4)}},
        "gpu_launches": steps * (1 + ps.plan["select"][1] + ps.plan["attend"][1])}
    del ps
    torch.cuda.empty_cache()
    return out


def run_b200(args, world, rank, local):
    import landmark_guided_chunk_b200 as hsa

    dev = torch.device("cuda", local)
    pk = peaks()
    ps = PrefillSetup(args.workload, args.seed + rank, dev)
    p, prob, plan, ws = ps.p, ps.prob, ps.plan, ps.ws
    Q, K, V, W, L, O = ps.Q, ps.K, ps.V, ps.W, ps.L, ps.O
    idx, score, keff, st = ps.idx, ps.score, ps.keff, ps.st
    clocks = ClockSampler(local)
    ms_step, stage_ms, keff_sum, clk = ps.time_stages(args.steps, args.warmup, world, clocks)
    tokens_all = p.B * p.Tq * world
    value = tokens_all / (ms_step * 1e-3)

    # End to end through the C ABI on host buffers: each step is one hsa_forward_host call, which copies the
    # step's inputs up from page-locked host memory, runs the whole forward and copies O back down, on its own
    # stream.  Three calls are in flight on three streams (each with its own device buffer and workspace),
    # so one call's uploads overlap another's compute and download, as a caller streaming independent
    # sequences would run it.  The window holds one pipeline fill and drain (the first upload, the last
    # compute and download), spread over the sequences it times; the steady state is bound by the uploads.
    nbuf = 3
    Qh, Kh, Vh, Wh = (x.cpu().pin_memory() for x in (Q, K, V, W))
    Ohs = [torch.empty(O.shape, dtype=O.dtype, pin_memory=True) for _ in range(nbuf)]
    devs = [torch.empty(hsa.forward_host_bytes(prob), dtype=torch.uint8, device=dev) for _ in range(nbuf)]
    wss = [ws] + [hsa.alloc_workspace(prob, dev) for _ in range(nbuf - 1)]
    sts = [torch.cuda.Stream(dev) for _ in range(nbuf)]
    e2e_steps = 24

    def run_e2e(nsteps):
        for i in range(nsteps):
            j = i % nbuf
            hsa.forward_host(Qh, Kh, Vh, Wh, p.S, p.k, p.tau, p.q_pos0, O=Ohs[j], dev=devs[j], ws=wss[j],
                             stream=sts[j])

    run_e2e(nbuf)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for s in sts:
        s.wait_event(e0)   # the first upload starts inside the timed region
    run_e2e(e2e_steps)
    for s in sts:
        fin = torch.cuda.Event()
        fin.record(s)
        st.wait_event(fin)
    e1.record(st)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    for w_ in wss:
        hsa.device_status(w_)
    h2d = sum(x.numel() * x.element_size() for x in (Qh, Kh, Vh, Wh))
    d2h = Ohs[0].numel() * Ohs[0].element_size()
    del Qh, Kh, Vh, Wh, Ohs, devs, wss

    stages_out, roof = ps.roofline(stage_ms, keff_sum, pk)
    launches = args.steps * (plan["landmarks"][1] + plan["select"][1] + plan["attend"][1])

    out = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": f"{p.name}: B{p.B} T{p.Tq} H{p.H} Hkv{p.Hkv} d{p.d} S{p.S} k{p.k}",
                      "global_batch": p.B * world, "seq_len": p.Tq, "parallelism": f"dp{world} (one sequence per GPU)",
                      "l2": "inputs larger than L2 (Q 512 MiB, K and V 128 MiB each); no flush"},
           "e2e": {"value": round(tokens_all / (e2e_ms * 1e-3), 1), "unit": "tokens/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3),
                   "call": "hsa_forward_host (page-locked host buffers; each call copies its inputs up, runs the "
                           "forward and copies O down on its stream)",
                   "pipelining": f"{e2e_steps} independent sequences, {nbuf} calls in flight on {nbuf} streams "
                                 "(own device buffer and workspace each); the window includes the pipeline's "
                                 "fill and drain"},
           "gpu_launches": launches, "roofline": roof, "stages": stages_out, "clocks": clk,
           "keff_mean": round(keff_sum / (p.B * p.Tq * p.Hkv), 3)}
    if not args.no_backward:
        out["backward"] = run_backward(args, p, hsa, Q, K, V, W, L, idx, score, keff, keff_sum, st, world)
    del ps, Q, K, V, W, L, O, idx, score, keff, ws
    torch.cuda.empty_cache()
    if not args.no_router and args.workload == "prefill_bf16":
        out["router_bf16"] = run_router(args, world, rank, local, pk)
    if not args.no_d64 and args.workload == "prefill_bf16":
        out["prefill_bf16_d64"] = run_prefill_line(args, world, rank, local, pk, "prefill_bf16_d64")
    if not args.no_variants and args.workload == "prefill_bf16":
        out["variants"] = run_variants(args, world, rank, local, pk)
    if not args.no_decode:
        out["decode_1m"] = run_decode(args, world, rank, local, pk)
        if not args.no_decode_16m:
            out["decode_16m"] = run_decode(args, world, rank, local, pk, "decode_16m")
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(p, args.seed)
    return out


# fp32 FMA peak of the CUDA cores: 148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz (clocks.max.sm)
FFMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_backward(args, p, hsa, Q, K, V, W, L, idx, score, keff, keff_sum, st, world):
    """hsa_backward on the forward's selection: dQ, dK, dV, dW_L (fp32) for a
    seeded upstream gradient dO.  Algorithmic work: the five S x d contractions
    per kept (query head, chunk) pair (Q K^T, dO V^T, dZ K, dZ^T Q, (wP)^T dO),
    2 S d FLOPs each."""
    from landmark_guided_chunk_b200.inputs import make_output_grad
    dev = Q.device
    dO = make_output_grad(p, seed=args.seed + 1000, device=dev)
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, Q.dtype)
    ws = torch.empty(hsa.backward_workspace_size(prob), dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = (torch.empty(Q.shape, **f32), torch.empty(K.shape, **f32), torch.empty(K.shape, **f32),
           torch.empty(p.d, p.d, **f32))

    from landmark_guided_chunk_b200 import dp

    def step():
        # each rank differentiates its own sequence; W_L's gradient is summed over the ranks
        dp.backward_dp(Q, K, V, W, L, idx, score, keff, dO, p.S, p.k, p.tau, q_pos0=p.q_pos0, out=out, ws=ws)

    for _ in range(max(3, args.warmup)):
        step()
    nsteps = max(1, min(args.steps, 5))
    barrier(world)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(nsteps):
        step()
    e1.record(st)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1) / nsteps, world)
    flops = 10.0 * p.S * p.d * p.G * float(keff_sum)
    ach = flops / (ms * 1e-3) / 1e12
    del ws, out, dO
    tc = p.dtype == "bf16" and p.d == 128 and p.S in (64, 128)
    pk = peaks()
    roof = ({"bound": "tensor", "achieved": round(ach, 2), "unit": "TFLOP/s", "peak": pk["bf16_tflops_sustained"],
             "frac": round(ach / pk["bf16_tflops_sustained"], 4),
             "peak_source": f"{pk['source']} (sustained bf16); whole backward call, 7 kernels"} if tc else
            {"bound": "alu", "achieved": round(ach, 2), "unit": "TFLOP/s", "peak": round(FFMA_PEAK_TFLOPS, 1),
             "frac": round(ach / FFMA_PEAK_TFLOPS, 4),
             "peak_source": "fp32 FMA lanes x clocks.max.sm (CUDA-core path)"})
    return {"ms": round(ms, 3), "steps": nsteps, "tokens_per_s": round(p.B * p.Tq * world / (ms * 1e-3), 1),
            "kernels": 7, "path": "tensor" if tc else "simt",
            "exchange": "all-reduce (sum) of dW_L, d x d fp32, over the ranks" if world > 1 else "none (one rank)",
            "dtype": "bf16 operands, fp32 accumulation" if tc else "f32", "roofline": roof}


def run_decode(args, world, rank, local, pk, name="decode_1m"):
    """One decode step (decode_1m: batch 8 at 1M context; decode_16m: batch 1 at
    16M context): landmarks precomputed, L2 flushed before each step, each step
    timed alone."""
    import landmark_guided_chunk_b200 as hsa
    from landmark_guided_chunk_b200.inputs import make_inputs, workload

    dev = torch.device("cuda", local)
    p = workload(name)
    inp = make_inputs(p, seed=args.seed + rank, device=dev)
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    L = hsa.landmarks(K, W, p.S)
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, torch.bfloat16,
                            hsa._native.HSA_FLAG_LANDMARKS_READY)
    plan = hsa.plan(prob)
    ws = hsa.alloc_workspace(prob, dev)
    O = torch.empty_like(Q)
    scrub = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def flush_l2():
        # write a buffer four times the L2 size, then read it back: the write
        # evicts everything else, the read leaves only clean lines behind, so
        # the timed kernels pay no write-back of the flush's dirty lines
        scrub.fill_(1)
        scrub.view(torch.int64).sum()
    st = torch.cuda.current_stream(dev)
    steps = max(args.steps, 10)

    def step():
        hsa.forward(Q, K, V, None, p.S, p.k, p.tau, p.q_pos0, L=L, landmarks_ready=True, O=O, ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    times = []
    for _ in range(steps):
        flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        step()
        b.record(st)
        b.synchronize()
        times.append(a.elapsed_time(b))
    torch.cuda.synchronize(dev)
    barrier(world)
    us = max_over_ranks(1e3 * statistics.median(times), world)
    # the two stages alone, each after an L2 scrub: scoring scan, and the chunk gather + fusion
    idx, sc, ke = hsa.select(Q, L, p.S, p.k, p.tau, p.q_pos0, Tkv=p.Tkv, ws=ws)
    sel_t, att_t = [], []
    for _ in range(steps):
        for lst, fn in ((sel_t, lambda: hsa.select(Q, L, p.S, p.k, p.tau, p.q_pos0, Tkv=p.Tkv, ws=ws)),
                        (att_t, lambda: hsa.attend(Q, K, V, idx, sc, ke, p.S, p.k, p.tau, p.q_pos0, O=O, ws=ws))):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            b.synchronize()
            lst.append(a.elapsed_time(b))
    # the gather kernel's own duration: NSEL calls back to back, each on the selection of a different random
    # query batch, so every call gathers chunks the others did not (the cache is 32 GiB, L2 126 MB) while
    # the host launch latency of one call overlaps the previous one
    NSEL = 8
    gsel = torch.Generator(device=dev).manual_seed(args.seed + 1000 + rank)
    qs = [torch.randn(Q.shape, device=dev, generator=gsel).to(Q.dtype) for _ in range(NSEL)]
    sels = [hsa.select(q, L, p.S, p.k, p.tau, p.q_pos0, Tkv=p.Tkv) for q in qs]
    outs = [torch.empty_like(Q) for _ in range(NSEL)]
    seq_t = []
    for _ in range(steps):
        flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for q, (si, ss, sk), o in zip(qs, sels, outs):
            hsa.attend(q, K, V, si, ss, sk, p.S, p.k, p.tau, p.q_pos0, O=o, ws=ws)
        b.record(st)
        b.synchronize()
        seq_t.append(a.elapsed_time(b) / NSEL)
    seq_bytes = sum(int(sk.long().sum().item()) for (_, _, sk) in sels) * p.S * p.d * 2 * 2 // NSEL
    hsa.device_status(ws)
    sel_us = max_over_ranks(1e3 * statistics.median(sel_t), world)
    att_us = max_over_ranks(1e3 * statistics.median(att_t), world)
    seq_us = max_over_ranks(1e3 * statistics.median(seq_t), world)
    # compulsory HBM bytes of one decode step: the landmark scan plus the k_eff chunks' K and V per (b, kv head)
    scan = p.B * p.Hkv * p.C * p.d * 2
    gather = int(ke.long().sum().item()) * p.S * p.d * 2 * 2
    gbs = (scan + gather) / (us * 1e-6) * 1e-9
    stages = {
        "select": {"us": round(sel_us, 2), "bytes": scan, "achieved_gbs": round(scan / (sel_us * 1e-6) * 1e-9, 1),
                   "frac": round(scan / (sel_us * 1e-6) * 1e-9 / pk["hbm_gbs"], 4)},
        "gather": {"us": round(seq_us, 2), "bytes": seq_bytes,
                   "achieved_gbs": round(seq_bytes / (seq_us * 1e-6) * 1e-9, 1),
                   "frac": round(seq_bytes / (seq_us * 1e-6) * 1e-9 / pk["hbm_gbs"], 4),
                   "timing": f"mean of {NSEL} back-to-back calls on {NSEL} different selections after one L2 flush",
                   "single_call_us": round(att_us, 2),
                   "single_call_timing": "one call after an L2 flush, incl. its status memset and launch"},
    }
    res = {"workload": f"{name}: B{p.B} ctx {p.Tkv} H{p.H} Hkv{p.Hkv} d{p.d} S{p.S} k{p.k}",
           "us_per_step": round(us, 2), "us_per_token": round(us / p.B, 3),
           "tokens_per_s": round(p.B * world / (us * 1e-6), 1),
           "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": round(gbs / pk["hbm_gbs"], 4), "bytes_per_step": scan + gather},
           "stages": stages,
           "l2": "512 MiB written then read before every step and before each stage timed alone", "paths": plan,
           "gpu_launches_per_step": plan["select"][1] + (0 if plan["forward_fused"] else plan["attend"][1]),
           "fused": ("one cooperative launch: the scan, then each row's chunk gather as soon as its selection "
                     "is published; the stages above are the same work as two separate calls")
           if plan["forward_fused"] else None}
    if name == "decode_1m":
        res["loop"] = decode_loop(p, hsa, Q, K, V, W, L, O, ws, st, world)
    if name == "decode_16m" and p.B == 1:
        res["sharded_8"] = sharded_share(p, hsa, Q, K, V, L, flush_l2, st, world)
    del inp, Q, K, V, W, L, O, ws, scrub, qs, sels, outs
    torch.cuda.empty_cache()
    return res


def sharded_share(p, hsa, Q, K, V, L, flush_l2, st, world, nshard=8):
    """One rank's share of a context-sharded decode step with the context split
    8 ways (landmark_guided_chunk_b200.sharded): the local selection and partial
    outputs over 1/8 of the cache, then the merge of 8 ranks' partials (this
    rank's, re-indexed as 8 disjoint chunk ranges).  The all-gather between them
    is not part of it: one GPU per run here."""
    from landmark_guided_chunk_b200 import sharded
    C = p.C
    c1 = C // nshard
    Kg, Vg = K[:, :c1 * p.S], V[:, :c1 * p.S]            # contiguous: B = 1
    Lg = L[:, :, :c1].contiguous()
    prob = hsa.make_problem(p.B, 1, c1 * p.S, p.H, p.Hkv, p.d, p.S, hsa.kmax_of(p.k, p.tau), c1 * p.S, 0.0,
                            torch.bfloat16)
    wsg = hsa.alloc_workspace(prob, Q.device)
    parts = sharded.shard_partials(Q, Kg, Vg, Lg, p.S, p.k, p.tau, p.Tkv, 0, ws=wsg)
    sc, gi, ke, o = parts
    stacked = (sc.unsqueeze(0).repeat(nshard, 1, 1, 1, 1),
               torch.stack([torch.where(gi >= 0, gi + s * c1, gi) for s in range(nshard)]),
               ke.unsqueeze(0).repeat(nshard, 1, 1, 1), o.unsqueeze(0).repeat(nshard, 1, 1, 1, 1, 1, 1))
    ts = {"local": [], "merge": []}
    for _ in range(10):
        flush_l2()
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(st)
        sharded.shard_partials(Q, Kg, Vg, Lg, p.S, p.k, p.tau, p.Tkv, 0, ws=wsg)
        b.record(st)
        hsa.merge_partials(*stacked, p.S, p.k, p.tau, dtype=Q.dtype)
        c.record(st)
        c.synchronize()
        ts["local"].append(a.elapsed_time(b) * 1e3)
        ts["merge"].append(b.elapsed_time(c) * 1e3)
    # back to back: the host's launches run ahead of the device, so this is device time
    NB = 10
    bb = []
    for _ in range(3):
        flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(NB):
            sharded.shard_partials(Q, Kg, Vg, Lg, p.S, p.k, p.tau, p.Tkv, 0, ws=wsg)
            hsa.merge_partials(*stacked, p.S, p.k, p.tau, dtype=Q.dtype)
        b.record(st)
        b.synchronize()
        bb.append(a.elapsed_time(b) * 1e3 / NB)
    hsa.device_status(wsg)
    loc = max_over_ranks(statistics.median(ts["local"]), world)
    mrg = max_over_ranks(statistics.median(ts["merge"]), world)
    b2b = max_over_ranks(statistics.median(bb), world)
    return {"nshard": nshard, "shard_tokens": c1 * p.S, "us_per_step_per_rank": round(b2b, 2),
            "single_local_us": round(loc, 2), "single_merge_us": round(mrg, 2),
            "exchange": f"not measured (one GPU per run): an all-gather of {nshard} x "
                        f"{(sc.numel() * 8 + ke.numel() * 4 + o.numel() * 4) // 1024} KiB",
            "timing": f"us_per_step_per_rank: mean of {NB} back-to-back (local + merge) after one L2 flush, median "
                      "of 3; single_*: one call each after an L2 flush, host launch latency included.  local = "
                      "selection (k = kmax, router off) + partial outputs over 1/8 of the chunks; merge = 8 ranks' "
                      "partials into O"}


def decode_loop(p, hsa, Q, K, V, W, L, O, ws, st, world):
    """A generation loop over the cache's last chunk: the cache starts S tokens short,
    and each step appends one token per sequence (hsa_decode_append; the S-th append
    completes the chunk and computes its landmark) and runs the forward of the next
    query on Tkv + 1 cached tokens.  The appended rows are the cache's own, so every
    step reads the same data as the one-step measurement.  Timed back to back (a
    running loop's steady state, no flush): whole steps, then the same forwards alone."""
    T0 = p.Tkv - p.S
    kn = [K[:, t].contiguous() for t in range(T0, p.Tkv)]
    vn = [V[:, t].contiguous() for t in range(T0, p.Tkv)]

    def run(append):
        for i in range(p.S):
            kv = T0 + i
            if append:
                hsa.decode_append(K, V, kn[i], vn[i], kv, p.S, W, L)
            hsa.forward(Q, K, V, None, p.S, p.k, p.tau, kv + 1, L=L, landmarks_ready=True, O=O, ws=ws,
                        kv_len=kv + 1)

    run(True)
    torch.cuda.synchronize()
    times = {}
    for label, app in (("step", True), ("forward", False)):
        ts = []
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            run(app)
            b.record(st)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e3 / p.S)
        times[label] = max_over_ranks(statistics.median(ts), world)
    hsa.device_status(ws)
    return {"us_per_step": round(times["step"], 2), "steps": p.S,
            "forward_only_us_per_step": round(times["forward"], 2),
            "append_us_per_step": round(times["step"] - times["forward"], 2),
            "timing": f"{p.S} steps back to back (no flush between them), median of 3 runs: append + forward, "
                      "then the same forwards alone; the append's cost is the difference (it includes the "
                      "one step in S that computes the completed chunk's landmark)"}


def dram_traffic(stage: str, path: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary,
    if it was taken on the kernel source that is built now; else None."""
    f = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(f) as fh:
            d = json.load(fh)
    except (OSError, ValueError):
        return None
    ent = d.get(f"{stage}:{path}")
    if not ent:
        return None
    if source_digest(ent.get("sources", [])) != ent.get("source_hash"):
        return None
    return ent.get("bytes_per_launch")


def source_digest(paths) -> str:
    """Digest of the code in the given source files, with // comments and blank
    lines left out: a capture stays valid across comment-only edits, and any
    change to the code itself invalidates it."""
    import hashlib
    import re
    h = hashlib.sha256()
    for src in paths:
        with open(os.path.join(ROOT, src)) as fh:
            for line in fh:
                code = re.sub(r"//.*$", "", line).rstrip()
                if code.strip():
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


# --------------------------------------------------------------------------- CPU baseline (oracle)

def _sample_positions(p, n, seed):
    rng = np.random.default_rng(seed)
    edges = np.linspace(0, p.Tq, n + 1).astype(np.int64)
    return np.array([rng.integers(edges[i], max(edges[i] + 1, edges[i + 1])) for i in range(n)])


def cpu_baseline(p, seed, n_tokens=None, budget_s=20.0):
    """The oracle, as it stands, on a bounded sample of the same workload: the
    landmarks of every chunk (timed), then selection + attention + fusion for
    n_tokens positions spread evenly over the sequence (all kv heads).  The
    throughput is tokens / (time per token of the rows + landmark time per
    token)."""
    import oracle
    from landmark_guided_chunk_b200.inputs import make_inputs

    inp = make_inputs(p, seed=seed, device="cpu")
    K, W = inp["K"], inp["W_L"]
    t0 = time.perf_counter()
    L = oracle.landmarks_stored(K, W, p.S, p.dtype)
    t_lm = time.perf_counter() - t0
    if n_tokens is None:
        # size the row sample from a short probe so the whole baseline stays near budget_s
        probe = _sample_positions(p, 8, seed)
        t0 = time.perf_counter()
        oracle.forward_rows(inp["Q"], K, inp["V"], W, p.S, p.k, p.tau, p.q_pos0, np.zeros(8, int), probe, L=L)
        per = (time.perf_counter() - t0) / 8
        n_tokens = int(max(16, min(4096, (budget_s - t_lm) / max(per, 1e-6))))
    pos = _sample_positions(p, n_tokens, seed + 1)
    t0 = time.perf_counter()
    oracle.forward_rows(inp["Q"], K, inp["V"], W, p.S, p.k, p.tau, p.q_pos0, np.zeros(n_tokens, int), pos, L=L)
    t_rows = time.perf_counter() - t0
    per_token = t_rows / n_tokens + t_lm / (p.B * p.Tq)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(1.0 / per_token, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"landmarks of all {p.B * p.C} chunks ({t_lm:.2f} s) + selection/attention/fusion of "
                      f"{n_tokens} positions spread over the sequence, all {p.Hkv} kv heads ({t_rows:.2f} s)"}


def run_reference(args, world, rank):
    """The oracle as the reference arm: each step processes S sampled query
    positions (all kv heads) plus the landmarks of one chunk of keys."""
    import oracle
    from landmark_guided_chunk_b200.inputs import make_inputs, workload

    p = workload(args.workload)
    inp = make_inputs(p, seed=args.seed, device="cpu")
    K, W = inp["K"], inp["W_L"]
    L = oracle.landmarks_stored(K, W, p.S, p.dtype)
    rng = np.random.default_rng(args.seed)

    def step():
        c = int(rng.integers(0, p.C))
        oracle.landmarks_stored(K[:, c * p.S:(c + 1) * p.S], W, p.S, p.dtype)
        pos = np.sort(rng.integers(0, p.Tq, p.S))
        oracle.forward_rows(inp["Q"], K, inp["V"], W, p.S, p.k, p.tau, p.q_pos0, np.zeros(p.S, int), pos, L=L)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = p.S / dt
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = (f"per step: {p.S} uniformly drawn query positions of {p.name} (all {p.Hkv} kv heads: selection, "
              f"attention, fusion) + the landmarks of one chunk")
    return {"metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": f"{p.name}: B{p.B} T{p.Tq} H{p.H} Hkv{p.Hkv} d{p.d} S{p.S} k{p.k}",
                       "global_batch": p.B, "seq_len": p.Tq, "parallelism": "cpu (oracle, all host cores)"},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}



# --------------------------------------------------------------------------- single-case driver for profilers

def run_case(args):
    """One workload (optionally resized) run --iters times through the public
    API, for profiler captures of a small, reproducible case:
      --T N         prefill length (Tq = Tkv = N)
      --ctx N       decode context length
      --B N         batch
      --select-only selection stage alone on the workload's query shapes and
                    random landmarks, no K/V allocated
      --backward    one forward (with its selection), then the backward --iters times
      --simt        CUDA-core kernels only (HSA_FLAG_SIMT)
    Prints the kernel path of each stage and the wall time of the last iteration."""
    import landmark_guided_chunk_b200 as hsa
    from landmark_guided_chunk_b200.inputs import make_inputs, make_output_grad, workload

    p = workload(args.workload)
    if args.B is not None:
        p = p.with_(B=args.B)
    if args.T is not None:
        p = p.with_(Tq=args.T, Tkv=args.T)
    if args.ctx is not None:
        p = p.with_(Tkv=args.ctx, q_pos0=args.ctx)
    torch.cuda.set_device(0)
    dt = torch.bfloat16 if p.dtype == "bf16" else torch.float32
    simt = hsa._native.HSA_FLAG_SIMT if args.simt else 0

    def timed(f):
        for _ in range(args.iters):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            f()
            torch.cuda.synchronize()
            last = time.perf_counter() - t0
        return last * 1e3

    if args.select_only:
        g = torch.Generator(device="cuda").manual_seed(0)
        Q = torch.randn(p.B, p.Tq, p.H, p.d, device="cuda", generator=g).to(dt)
        L = (torch.randn(p.B, p.Hkv, p.C, p.d, device="cuda", generator=g) / 8).to(dt)
        prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, dt, simt)
        ws = hsa.alloc_workspace(prob)
        ms = timed(lambda: hsa.select(Q, L, p.S, p.k, p.tau, p.q_pos0, Tkv=p.Tkv, ws=ws, force_simt=args.simt))
        hsa.device_status(ws)
        print(f"{p.name} (select only): B{p.B} Tq{p.Tq} Tkv{p.Tkv} plan={hsa.plan(prob)} last={ms:.3f} ms")
        return
    inp = make_inputs(p, seed=0, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    if args.backward:
        O, L, idx, sc, ke = hsa.forward(Q, K, V, W, p.S, p.k, p.tau, p.q_pos0, return_selection=True)
        dO = make_output_grad(p, seed=1, device="cuda")
        prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, dt, simt)
        ws = torch.empty(hsa.backward_workspace_size(prob), dtype=torch.uint8, device="cuda")
        f32 = dict(dtype=torch.float32, device="cuda")
        out = (torch.empty(Q.shape, **f32), torch.empty(K.shape, **f32), torch.empty(K.shape, **f32),
               torch.empty(p.d, p.d, **f32))
        ms = timed(lambda: hsa.backward(Q, K, V, W, L, idx, sc, ke, dO, p.S, p.k, p.tau, p.q_pos0, out=out, ws=ws,
                                        force_simt=args.simt))
        hsa.device_status(ws)
        print(f"{p.name} backward: B{p.B} Tq{p.Tq} Tkv{p.Tkv} simt={args.simt} last={ms:.3f} ms")
        return
    ready = p.is_decode
    L = hsa.landmarks(K, W, p.S) if ready else None
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, dt,
                            (hsa._native.HSA_FLAG_LANDMARKS_READY if ready else 0) | simt)
    ws = hsa.alloc_workspace(prob)
    O = torch.empty_like(Q)
    ms = timed(lambda: hsa.forward(Q, K, V, None if ready else W, p.S, p.k, p.tau, p.q_pos0, L=L,
                                   landmarks_ready=ready, O=O, ws=ws, force_simt=args.simt))
    hsa.device_status(ws)
    print(f"{p.name}: B{p.B} Tq{p.Tq} Tkv{p.Tkv} plan={hsa.plan(prob)} last={ms:.3f} ms")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default="prefill_bf16",
                    help="prefill_bf16 | router_bf16 | tiny_f32 (with --case also decode_1m, decode_16m)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-decode-16m", action="store_true", help="skip the 16M-context decode line (64 GiB cache)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass line")
    ap.add_argument("--no-router", action="store_true", help="skip the gap-router prefill line (router_bf16)")
    ap.add_argument("--no-variants", action="store_true", help="skip the selection-variant lines (Quest, refiner)")
    ap.add_argument("--no-d64", action="store_true", help="skip the head-dim-64 prefill line (prefill_bf16_d64)")
    ap.add_argument("--case", action="store_true",
                    help="single-case driver for profiler captures (see run_case); prints no JSON line")
    ap.add_argument("--iters", type=int, default=3, help="--case: iterations")
    ap.add_argument("--T", type=int, default=None, help="--case: prefill length (Tq = Tkv)")
    ap.add_argument("--ctx", type=int, default=None, help="--case: decode context length")
    ap.add_argument("--B", type=int, default=None, help="--case: batch")
    ap.add_argument("--simt", action="store_true", help="--case: CUDA-core kernels only")
    ap.add_argument("--select-only", action="store_true", help="--case: selection stage only, random landmarks")
    ap.add_argument("--backward", action="store_true", help="--case: one forward, then the backward --iters times")
    args = ap.parse_args()
    if args.case:
        run_case(args)
        return
    if args.workload not in ("prefill_bf16", "router_bf16", "tiny_f32"):
        ap.error(f"--workload {args.workload} is a --case workload; the bench line runs a prefill workload")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world, rank)), flush=True)
        return
    world, rank, local = dist_setup()
    out = run_b200(args, world, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
