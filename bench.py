"""Benchmark of the speculative-decoding verify step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--sigma S]
                    [--impl {mtpv,reference}] [--no-cpu-baseline] [--no-e2e] [--no-graph]
                    [--no-extra]
    python bench.py --proj     (int4 decoder-layer projections at small M)

One step = the whole verify step of one batch: the K+1 target rows through
the bf16 LM head, the K draft rows through the int4 group-64 head, and the
Leviathan-Chen verification (acceptance, residual / bonus draw).  Inputs are
seeded synthetic tensors with the shapes of a Qwen-class 27B model (hidden
5120, vocabulary 151936; random-init heads W ~ N(0, 0.02^2)), resident in HBM
before timing.  The heads (1.98 GB per step) are far larger than L2, so every
step streams them from HBM.

Multi-GPU: the verify step does not shard; N ranks run N independent
replicas (weak scaling) and the time is the max over ranks.

Prints one JSON line (rank 0).  Besides the headline workload (hidden 5120,
vocabulary 151936, K = 3), a one-GPU run adds three keys, each timed the
same way on its own synthetic inputs: "sweep" (draft depth K in {1, 2, 3} x
T in {0.6, 0} x draft noise sigma in {0.1, 0.3, 1.0}: step time spread and
acceptance per cell), "large_vocab_b8" (8 sequences, vocabulary 248320) and
"projections" (the int4 decoder-layer projections at M = 1..8).
"""
from __future__ import annotations

import argparse
import json
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

from verify_step_lm_b200 import synth  # noqa: E402

CONFIGS = {
    # name: B, K, V, h, T, top_p, draft noise sigma, head std
    "qwen27b": dict(B=1, K=3, V=151936, h=5120, T=0.6, top_p=0.95, sigma=0.3, wstd=0.02),
    "qwen27b_k1": dict(B=1, K=1, V=151936, h=5120, T=0.6, top_p=0.95, sigma=0.3, wstd=0.02),
    "qwen27b_k2": dict(B=1, K=2, V=151936, h=5120, T=0.6, top_p=0.95, sigma=0.3, wstd=0.02),
    "qwen27b_greedy": dict(B=1, K=3, V=151936, h=5120, T=0.0, top_p=0.95, sigma=0.3, wstd=0.02),
    "b8_v248k": dict(B=8, K=3, V=248320, h=5120, T=0.6, top_p=0.95, sigma=0.3, wstd=0.02),
    "tiny": dict(B=1, K=3, V=4096, h=512, T=0.6, top_p=0.95, sigma=0.3, wstd=0.05),
}
POOL = 64
SWEEP_K, SWEEP_T, SWEEP_SIGMA = (1, 2, 3), (0.6, 0.0), (0.1, 0.3, 1.0)
METRIC = "verify steps/s (K=3, V=151936, h=5120) and achieved HBM GB/s vs roofline"


def recorded_traffic(kernel_source: str, profile: str):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel's source changed since the counters were taken."""
    import hashlib
    try:
        text = open(os.path.join(ROOT, "profiles", profile)).read()
        line = next(l for l in text.splitlines() if "traffic_bytes_per_launch=" in l)
        f = dict(kv.split("=", 1) for kv in line.split())
        src = open(os.path.join(ROOT, kernel_source), "rb").read()
        if f.get("sha256") != hashlib.sha256(src).hexdigest():
            return None
        return int(f["traffic_bytes_per_launch"])
    except Exception:
        return None


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def workload_name(c):
    return (f"verify step B={c['B']} K={c['K']} hidden={c['h']} vocab={c['V']}: bf16 target head + "
            f"int4 g64 draft head + Leviathan-Chen sampler, T={c['T']}, top_p={c['top_p']}")


def step_bytes(c):
    """Algorithmic HBM bytes of one step: both heads once, hidden states, the
    fp32 logits written by the heads and read once by the sampler."""
    B, K, V, h = c["B"], c["K"], c["V"], c["h"]
    Mt, Md = B * (K + 1), B * K
    w_bf16 = V * h * 2
    w_int4 = V * h // 2 + V * (h // 64) * 2
    hidden = (Mt + Md) * h * 2
    logits = (Mt + Md) * V * 4
    return {"w_bf16": w_bf16, "w_int4": w_int4, "hidden": hidden, "logits_rw": 2 * logits,
            "bf16_launch": w_bf16 + Mt * h * 2 + Mt * V * 4,
            "int4_launch": w_int4 + Md * h * 2 + Md * V * 4,
            "sampler_launch": logits,
            "total": w_bf16 + w_int4 + hidden + 2 * logits}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# ---------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_steps(c, seconds: float, min_steps: int, max_steps: int, heads=None):
    """Time the CPU oracle on whole verify steps of workload c (host cores).

    ``heads`` = (W, Wq, S) CPU tensors to reuse; generated here otherwise.
    """
    import oracle  # test infrastructure: used here only for the CPU baseline

    B, K, V, h = c["B"], c["K"], c["V"], c["h"]
    T32, P32 = float(np.float32(c["T"])), float(np.float32(c["top_p"]))
    cores = host_cores()
    if heads is None:
        W = synth.make_head(V, h, c["wstd"], seed=12345)
        Wq, S = synth.quantize_int4_g64(W)
    else:
        W, Wq, S = heads
    Wb, Wqn, Sb = synth.bf16_bits(W), Wq.numpy(), synth.bf16_bits(S)
    elapsed, steps = 0.0, 0
    while steps < max_steps and (steps < min_steps or elapsed < seconds):
        Ht, Hd = synth.make_hidden(B, K, h, c["sigma"], seed=1000 + steps)
        u = synth.step_uniforms(1000 + steps, 0, B, K)
        # drafts from the oracle's own q' (input preparation, not timed)
        dl0 = oracle.lm_head_int4g64(synth.bf16_bits(Hd), Wqn, Sb, threads=cores)
        d, _, _ = oracle.sample_rows(dl0, T32, P32, u["u_draft"].reshape(-1), threads=cores)
        t0 = time.perf_counter()
        tl = oracle.lm_head_bf16(synth.bf16_bits(Ht), Wb, threads=cores)
        dl = oracle.lm_head_int4g64(synth.bf16_bits(Hd), Wqn, Sb, threads=cores)
        oracle.verify(tl.reshape(B, K + 1, V), dl.reshape(B, K, V), d.reshape(B, K), u["u_accept"],
                      u["u_sample"], T32, P32, threads=min(cores, B))
        elapsed += time.perf_counter() - t0
        steps += 1
    return steps, elapsed, cores


def run_reference(args, c, rank):
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_steps(c, 0.0, 1, 1)
    steps, elapsed, cores = oracle_steps(c, 0.0, args.steps, args.steps)
    v = steps / elapsed
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(c, args.config, args.gpus),
        "cpu_baseline": {"value": v, "unit": "steps/s", "cores": cores, "kind": "oracle",
                         "sample": f"{steps} whole verify steps of the workload, fp64 C oracle"},
        "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class Replicas:
    """Rank bookkeeping of an N-replica run: every rank runs the whole step on
    its own batch (the verify step does not shard), ranks meet at barriers
    around the timed region, the time is the max over ranks, and the
    whole-job value counts every rank's steps.  Works on any process group
    (NCCL with device tensors on the GPU machine, gloo with CPU tensors in the
    tests); with world == 1 nothing is exchanged."""

    def __init__(self, world: int, rank: int, device):
        self.world, self.rank, self.device = world, rank, device

    def barrier(self):
        if self.world > 1:
            torch.distributed.barrier()

    def max_over_ranks(self, x: float) -> float:
        if self.world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())

    def job_value(self, ms_per_step: float) -> float:
        """Steps per second of the whole job: world steps per max-over-ranks step time."""
        return self.world * 1e3 / ms_per_step


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def make_heads(c, dev):
    W = synth.make_head(c["V"], c["h"], c["wstd"], seed=12345, device=dev)
    Wq, S = synth.quantize_int4_g64(W)
    return W, Wq, S


def build_pool(c, dev, mtpv, heads, n=POOL, sigma=None):
    """n pre-generated steps: hidden states (draft noise sigma), uniforms, and
    drafts drawn by the library's own sampler from q' (the draft phase)."""
    B, K, V, h = c["B"], c["K"], c["V"], c["h"]
    W, Wq, S = heads
    sigma = c["sigma"] if sigma is None else sigma
    ht, hd, dr, ua, us = [], [], [], [], []
    dl = torch.empty((B * K, V), dtype=torch.float32, device=dev)
    for i in range(n):
        Ht, Hd = synth.make_hidden(B, K, h, sigma, seed=i, device=dev)
        u = synth.step_uniforms(i, 0, B, K)
        mtpv.lm_head_smallm(Hd, Wq, S, mtpv.W_INT4_G64, dl)
        d = torch.empty((B * K,), dtype=torch.int32, device=dev)
        mtpv.sample(dl, c["T"], c["top_p"], torch.as_tensor(u["u_draft"].reshape(-1)).to(dev), d)
        ht.append(Ht)
        hd.append(Hd)
        dr.append(d.view(B, K))
        ua.append(torch.as_tensor(u["u_accept"]).to(dev))
        us.append(torch.as_tensor(u["u_sample"]).to(dev))
    torch.cuda.synchronize()
    return ht, hd, dr, ua, us


def spread(ms):
    """median / p10 / p90 of per-step times (ms) in microseconds."""
    a = np.asarray(ms, dtype=np.float64) * 1e3
    return {"median": float(np.median(a)), "p10": float(np.percentile(a, 10)),
            "p90": float(np.percentile(a, 90)), "n": int(a.size)}


class StepRunner:
    """One workload on one device: heads, a pool of steps, output buffers and
    the workspace; step(i) runs pool entry i % n through mtpv_verify_step."""

    def __init__(self, c, dev, mtpv, heads=None, sigma=None, n=POOL):
        self.c, self.dev, self.mtpv = c, dev, mtpv
        B, K, V, h = c["B"], c["K"], c["V"], c["h"]
        self.heads = heads if heads is not None else make_heads(c, dev)
        self.pool = build_pool(c, dev, mtpv, self.heads, n=n, sigma=sigma)
        self.n = n
        self.tl = torch.empty((B, K + 1, V), dtype=torch.float32, device=dev)
        self.dl = torch.empty((B, K, V), dtype=torch.float32, device=dev)
        self.ot = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
        self.oa = torch.empty((B,), dtype=torch.int32, device=dev)
        self.rs = torch.empty((B,), dtype=torch.int32, device=dev)
        self.ws = mtpv.workspace(mtpv.verify_step_workspace_bytes(B, K, V, h), dev)
        self.stream = torch.cuda.current_stream(dev)

    def step(self, i):
        c, (W, Wq, S) = self.c, self.heads
        ht, hd, dr, ua, us = self.pool
        j = i % self.n
        self.mtpv.verify_step(W, Wq, S, ht[j], hd[j], dr[j], ua[j], us[j], c["B"], c["K"], c["T"],
                              c["top_p"], self.ot, self.oa, self.rs, self.tl, self.dl, self.ws)

    def timed(self, steps, barrier=lambda: None):
        """(mean ms per step over the whole region, per-step ms list): events
        on the launching stream after every step."""
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        barrier()
        torch.cuda.synchronize()
        ev[0].record(self.stream)
        for i in range(steps):
            self.step(i)
            ev[i + 1].record(self.stream)
        torch.cuda.synchronize()
        barrier()
        per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
        return ev[0].elapsed_time(ev[steps]) / steps, per

    def acceptance(self):
        """Accepted drafts over every pool step (untimed): rate = E[n] / K."""
        acc = []
        for j in range(self.n):
            self.step(j)
            acc.append(self.oa.clone())
        torch.cuda.synchronize()
        a = torch.cat(acc).double()
        K = self.c["K"]
        return {"rate": float(a.mean()) / K, "tokens_per_step": float(a.mean()) + 1.0,
                "all_accepted": float((a == K).double().mean()), "steps": self.n,
                "sequences": int(a.numel())}

    def breakdown(self, steps, barrier=lambda: None):
        """Mean ms of the heads launch and of the sampler, issued separately
        with events between them, for `steps` steps."""
        c, (W, Wq, S), mtpv = self.c, self.heads, self.mtpv
        B, K, V = c["B"], c["K"], c["V"]
        ht, hd, dr, ua, us = self.pool
        pws = mtpv.workspace(mtpv.load().mtpv_lm_head_pair_workspace_bytes(B * (K + 1), B * K, c["h"], V),
                             self.dev)
        vws = mtpv.workspace(mtpv.verify_workspace_bytes(B, K, V), self.dev)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            j = i % self.n
            evs[i][0].record(self.stream)
            mtpv.lm_head_pair(ht[j], W, self.tl.view(B * (K + 1), V), hd[j], Wq, S, self.dl.view(B * K, V),
                              ws=pws)
            evs[i][1].record(self.stream)
            mtpv.verify(self.tl, self.dl, dr[j], ua[j], us[j], c["T"], c["top_p"], self.ot, self.oa, self.rs,
                        ws=vws)
            evs[i][2].record(self.stream)
        torch.cuda.synchronize()
        barrier()
        heads = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
        samp = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        return heads, samp


def fused_heads(c):
    """Whether the step runs both heads in one launch (the two-head kernel)."""
    B, K, h = c["B"], c["K"], c["h"]
    return B * (K + 1) <= 8 and B * K <= 8 and h % 512 == 0 and \
        (2 * B * (K + 1) * (h + 32) + (B * K + 1) * (h // 8 + 1) * 16 + h // 2 + 3 * 13056) <= 227 * 1024 - 256


def config_dict(c, name, world):
    return {"workload": workload_name(c), "global_batch": c["B"] * world, "seq_len": c["K"] + 1,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"inputs larger than L2: {step_bytes(c)['w_bf16'] + step_bytes(c)['w_int4']:.3g} B of "
                  "head weights streamed per step",
            "config_name": name, "draft_noise_sigma": c["sigma"]}


def run_sweep(dev, mtpv, steps, warmup):
    """The draft-depth sweep at the Qwen-class heads: K in {1, 2, 3}, T in
    {0.6, 0 (greedy)}, draft noise sigma in {0.1, 0.3, 1.0}; per cell the
    step time (mean, median, p10, p90) and the acceptance over 64 steps."""
    base = CONFIGS["qwen27b"]
    heads = make_heads(base, dev)
    cells = []
    for K in SWEEP_K:
        for T in SWEEP_T:
            for sigma in SWEEP_SIGMA:
                c = dict(base, K=K, T=T, sigma=sigma)
                r = StepRunner(c, dev, mtpv, heads=heads)
                for i in range(warmup):
                    r.step(i)
                ms, per = r.timed(steps)
                acc = r.acceptance()
                cells.append({"K": K, "T": T, "sigma": sigma, "steps_per_s": 1e3 / ms, "ms_per_step": ms,
                              "step_us": spread(per), "acceptance": acc,
                              "tokens_per_s": (1e3 / ms) * acc["tokens_per_step"]})
                del r
    return {"workload": "hidden 5120, vocab 151936, B=1, top_p=0.95, head W ~ N(0, 0.02^2)",
            "steps_per_cell": steps, "cells": cells}


def run_extra_config(name, dev, mtpv, steps, warmup, peak):
    """Steps/s, per-step spread, kernel breakdown and heads roofline of one
    more workload (its own heads)."""
    c = CONFIGS[name]
    r = StepRunner(c, dev, mtpv)
    for i in range(warmup):
        r.step(i)
    ms, per = r.timed(steps)
    heads_ms, samp_ms = r.breakdown(steps)
    sb = step_bytes(c)
    hb = sb["bf16_launch"] + sb["int4_launch"]
    out = {"config": config_dict(c, name, 1), "steps_per_s": 1e3 / ms, "ms_per_step": ms,
           "step_us": spread(per), "kernels_ms": {"lm_heads": heads_ms, "sampler": samp_ms},
           "heads_roofline": {"achieved": hb / (heads_ms * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                              "frac": hb / (heads_ms * 1e-3) / 1e9 / peak, "algorithmic_bytes": hb},
           "step_roofline": {"achieved": sb["total"] / (ms * 1e-3) / 1e9, "peak": peak,
                             "frac": sb["total"] / (ms * 1e-3) / 1e9 / peak,
                             "algorithmic_bytes_per_step": sb["total"]},
           "acceptance": r.acceptance()}
    del r
    return out


def run_gpu(args, c, rank, world, local_rank):
    import verify_step_lm_b200 as mtpv

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    mtpv.load()
    B, K, V, h = c["B"], c["K"], c["V"], c["h"]
    T, top_p = c["T"], c["top_p"]
    r = StepRunner(c, dev, mtpv)
    W, Wq, S = r.heads
    fused = fused_heads(c)
    stream = r.stream
    reps = Replicas(world, rank, dev)
    barrier, max_over_ranks = reps.barrier, reps.max_over_ranks

    # --- warm-up
    for i in range(args.warmup):
        r.step(i)
    torch.cuda.synchronize()

    # --- timed region: K whole steps through the product entry point (an
    # event after every step gives the per-step spread)
    with ClockSampler(dev.index) as clk:
        step_ms, per_step = r.timed(args.steps, barrier)
        # per-kernel breakdown: the launches the step makes (both heads, then
        # the sampler's two kernels) with events between them
        k_heads, k_samp = r.breakdown(args.steps, barrier)
        # each head alone through its own kernel (reference for the fused launch)
        ht, hd = r.pool[0], r.pool[1]
        nalone = min(args.steps, 500)
        sev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nalone)]
        barrier()
        torch.cuda.synchronize()
        for i in range(nalone):
            j = i % POOL
            sev[i][0].record(stream)
            mtpv.lm_head_smallm(ht[j], W, None, mtpv.W_BF16, r.tl.view(B * (K + 1), V))
            sev[i][1].record(stream)
            mtpv.lm_head_smallm(hd[j], Wq, S, mtpv.W_INT4_G64, r.dl.view(B * K, V))
            sev[i][2].record(stream)
        torch.cuda.synchronize()
        barrier()
    clocks = clk.summary()
    k_bf16 = statistics.mean(e[0].elapsed_time(e[1]) for e in sev)
    k_int4 = statistics.mean(e[1].elapsed_time(e[2]) for e in sev)

    step_ms = max_over_ranks(step_ms)
    value = reps.job_value(step_ms)

    # --- the same steps replayed from CUDA graphs (one captured graph per
    # pool entry; the library makes no allocation or host sync inside a step)
    graph = None
    if not args.no_graph:
        graphs = []
        for j in range(POOL):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                r.step(j)
            graphs.append(g)
        torch.cuda.synchronize()
        for i in range(args.warmup):
            graphs[i % POOL].replay()
        barrier()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for i in range(args.steps):
            graphs[i % POOL].replay()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        graph_ms = max_over_ranks(g0.elapsed_time(g1) / args.steps)
        graph = {"value": reps.job_value(graph_ms), "unit": "steps/s", "ms_per_step": graph_ms,
                 "graphs": POOL, "nodes_per_step": f"{3 if fused else 4} kernels"}
        del graphs

    # --- end to end: host buffers through mtpv_verify_step_host
    e2e = None
    if not args.no_e2e:
        pin = lambda t: t.cpu().contiguous().pin_memory()
        hht, hhd, hdr, hua, hus = ([pin(x) for x in lst] for lst in r.pool)
        hot = torch.empty((B, K + 1), dtype=torch.int32).pin_memory()
        hoa = torch.empty((B,), dtype=torch.int32).pin_memory()
        hrs = torch.empty((B,), dtype=torch.int32).pin_memory()
        hws = mtpv.workspace(mtpv.verify_step_host_workspace_bytes(B, K, V, h), dev)

        def hstep(i):
            j = i % POOL
            mtpv.verify_step_host(W, Wq, S, hht[j], hhd[j], hdr[j], hua[j], hus[j], B, K, T, top_p,
                                  hot, hoa, hrs, hws)

        for i in range(args.warmup):
            hstep(i)
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(args.steps):
            hstep(i)
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1) / args.steps)
        h2d = (B * (K + 1) * h + B * K * h) * 2 + B * K * 4 + B * K * 4 + B * (K + 1) * 4
        d2h = B * (K + 1) * 4 + B * 4 + B * 4
        e2e = {"value": reps.job_value(e2e_ms), "unit": "steps/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "api": "mtpv_verify_step_host (pinned host inputs/outputs)"}

    acceptance = r.acceptance()
    if rank != 0:
        return
    peak, peak_kind = measured_peaks()
    sb = step_bytes(c)
    heads_bytes = sb["bf16_launch"] + sb["int4_launch"]
    achieved = heads_bytes / (k_heads * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16/int4 weights, fp32 accumulate, f64 sampler",
        "data": "synthetic",
        "config": config_dict(c, args.config, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": recorded_traffic("verify_step_lm_b200/csrc/lm_head.cu",
                                                 "lm_heads_mixed_qwen27b.md") if fused and
                                args.config == "qwen27b" and args.sigma is None else None,
                     "kernel": "lm_heads_mixed_kernel (both heads, one launch)" if fused
                               else "lm_head_bf16_mma_kernel + lm_head_int4_f16_kernel",
                     "algorithmic_bytes_per_launch": heads_bytes, "peak_source": peak_kind},
        "step_roofline": {"achieved": sb["total"] / (step_ms * 1e-3) / 1e9, "peak": peak,
                          "unit": "GB/s", "frac": sb["total"] / (step_ms * 1e-3) / 1e9 / peak,
                          "frac_of_8tbs": sb["total"] / (step_ms * 1e-3) / 8e12,
                          "algorithmic_bytes_per_step": sb["total"]},
        "step_us": spread(per_step),
        "kernels_ms": {"lm_heads": k_heads, "sampler": k_samp},
        "heads_alone_ms": {"lm_head_bf16": k_bf16, "lm_head_int4": k_int4,
                           "bf16_gbs": sb["bf16_launch"] / (k_bf16 * 1e-3) / 1e9,
                           "int4_gbs": sb["int4_launch"] / (k_int4 * 1e-3) / 1e9},
        "acceptance": acceptance,
        "gpu_launches": (3 if fused else 4) * args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "graph": graph,
    }
    if not args.no_extra and world == 1:
        del r
        torch.cuda.empty_cache()
        n = max(50, min(args.steps, 200))
        line["sweep"] = run_sweep(dev, mtpv, n, max(3, min(args.warmup, 10)))
        torch.cuda.empty_cache()
        line["large_vocab_b8"] = run_extra_config("b8_v248k", dev, mtpv, n, max(3, min(args.warmup, 10)), peak)
        torch.cuda.empty_cache()
        line["projections"] = run_proj(args, quiet=True)
    if not args.no_cpu_baseline and world == 1:
        steps, elapsed, cores = oracle_steps(c, seconds=10.0, min_steps=2, max_steps=30,
                                             heads=(W.cpu(), Wq.cpu(), S.cpu()))
        line["cpu_baseline"] = {"value": steps / elapsed, "unit": "steps/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"{steps} whole verify steps of the workload (fp64 C oracle, "
                                          f"{cores} threads), {elapsed:.1f} s"}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# decoder-layer projections (int4 g64, small M): a separate measurement mode
# ---------------------------------------------------------------------------
PROJ_SHAPES = [  # name, Kd, N (gate_up: N = 2F, output F)
    ("qkv", 5120, 7168), ("o", 5120, 5120), ("gate_up", 5120, 2 * 17408), ("down", 17408, 5120)]


def run_proj(args, quiet=False):
    """Each projection of a 27B-class decoder layer at M in {1..6, 8}, weights
    rotated over enough copies (>= 4x the L2) that every call streams them
    from HBM; CUDA-event time per call, plain launches and CUDA-graph replay.
    Prints one JSON line, or (quiet) returns it."""
    import verify_step_lm_b200 as mtpv

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    mtpv.load()
    peak, peak_kind = measured_peaks()
    layer_bytes = sum(N * (Kd // 2) + N * (Kd // 64) * 2 for _, Kd, N in PROJ_SHAPES)
    copies = max(2, -(-4 * 126 * 2 ** 20 // layer_bytes))
    layers = []
    for c in range(copies):
        lay = {}
        for name, Kd, N in PROJ_SHAPES:
            W = synth.make_head(N, Kd, 0.02, seed=700 + 10 * c + len(lay), device=dev)
            lay[name] = synth.quantize_int4_g64(W)
            del W
        layers.append(lay)
    stream = torch.cuda.current_stream(dev)
    out = {}
    for M in (1, 2, 3, 4, 5, 6, 8):
        row = {}
        for name, Kd, N in PROJ_SHAPES:
            x = synth.gaussian((M, Kd), 1.0, 900 + M, dev)
            ncols = N // 2 if name == "gate_up" else N
            y = torch.empty((M, ncols), dtype=torch.float32, device=dev)
            if name == "gate_up":
                ws = mtpv.workspace(mtpv.load().mtpv_int4_gate_up_workspace_bytes(M, Kd, N // 2), dev)
                call = lambda lay: mtpv.int4_gate_up(x, lay[name][0], lay[name][1], y, ws=ws)
            else:
                ws = mtpv.workspace(mtpv.load().mtpv_int4_proj_workspace_bytes(M, Kd, N), dev)
                call = lambda lay: mtpv.int4_proj(x, lay[name][0], lay[name][1], y, ws=ws)
            for i in range(args.warmup):
                call(layers[i % copies])
            n = max(30, min(args.steps, 400))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            for i in range(n):
                call(layers[i % copies])
            e1.record(stream)
            torch.cuda.synchronize()
            us = 1e3 * e0.elapsed_time(e1) / n
            graphs = []
            for c in range(copies):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    call(layers[c])
                graphs.append(g)
            for i in range(args.warmup):
                graphs[i % copies].replay()
            torch.cuda.synchronize()
            e0.record(stream)
            for i in range(n):
                graphs[i % copies].replay()
            e1.record(stream)
            torch.cuda.synchronize()
            us_graph = 1e3 * e0.elapsed_time(e1) / n
            del graphs
            nbytes = N * (Kd // 2) + N * (Kd // 64) * 2 + M * Kd * 2 + M * ncols * 4
            row[name] = {"us": us, "us_graph": us_graph, "gbs": nbytes / (us * 1e-6) / 1e9,
                         "frac": nbytes / (us * 1e-6) / 1e9 / peak, "bytes": nbytes}
        row["layer_us"] = sum(v["us"] for v in row.values() if isinstance(v, dict))
        row["layer_us_graph"] = sum(v["us_graph"] for k, v in row.items() if isinstance(v, dict))
        out[M] = row
    line = {"metric": "int4 g64 decoder-layer projections (qkv, o, gate||up with SiLU, down) per layer",
            "unit": "us", "higher_is_better": False, "n_gpus": 1, "data": "synthetic",
            "config": {"workload": "27B-class layer: hidden 5120, intermediate 17408, qkv 7168; "
                                   "W ~ N(0, 0.02^2) -> int4 g64, activations N(0,1) bf16",
                       "weight_copies": copies, "l2": "weights rotated over >= 4x L2"},
            "peak_gbs": peak, "peak_source": peak_kind, "by_m": out}
    del layers
    torch.cuda.empty_cache()
    if quiet:
        return line
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--config", default="qwen27b", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="mtpv", choices=["mtpv", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the depth sweep, the large-vocabulary batch and the projections")
    ap.add_argument("--sigma", type=float, default=None,
                    help="draft-noise sigma of the workload (sets the acceptance rate)")
    ap.add_argument("--proj", action="store_true",
                    help="time the int4 decoder-layer projections instead of the verify step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    c = dict(CONFIGS[args.config])
    if args.sigma is not None:
        c["sigma"] = args.sigma
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, c, rank)
        return
    if args.proj:
        if rank == 0:
            run_proj(args)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_gpu(args, c, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
