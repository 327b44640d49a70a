#!/usr/bin/env python
"""Benchmark of libgdn2 on B200: Gated DeltaNet-2 chunk-forward tokens/s (headline) and
decode tokens/s, each with its HBM roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {libgdn2,reference}]

A step is one gdn2_chunk_fwd over the prefill workload (batch 8, 16 heads, T=4096,
dk=dv=128, bf16 inputs, fp32 log-decay and state). A token is one position of one sequence
across all heads. Inputs (1.07 GB) are larger than L2, so no flush is needed between steps.
Under torchrun every rank runs its own batch (weak scaling, no collective on the data
path); the time is the maximum over ranks. Rank 0 prints one JSON line.

--impl reference times the oracle (fp64, CPU, OpenMP) on a bounded sample of the same
workload on this host's cores.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL = "prefill_b8_h16_t4096"
DECODE = "decode_256seq_h32"
GROUPED = "grouped_b2_qk16_v32_t32768"
GROUPED_TIMED_STEPS = 5
VARLEN = "varlen_64seq_h16"
VARLEN_TIMED_STEPS = 3
# fp32 SIMT peak for the backward's per-token adjoint: 148 SMs x 128 fp32 lanes x 2 flop
# (one FMA) per clock at the 1965 MHz maximum SM clock
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
SERVING_TOKENS = 4  # tokens per sequence in one serving-decode step (a verify step)
PROLOGUE_TIMED_STEPS = 10
BACKWARD_TIMED_STEPS = 3
DECODE_TIMED_STEPS = 512  # the decode workload's 512 consecutive steps
SERVING_TIMED_STEPS = 64


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libgdn2", choices=["libgdn2", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms while running."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.2)
        except FileNotFoundError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.1)
            self.proc.terminate()
            self.proc.wait(timeout=5)

    def summary(self, t_from=None, t_to=None):
        """Median SM clock, the max clock and the throttle reasons seen, over the samples that
        arrived between host times t_from and t_to (all samples by default)."""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, ln in self.lines:
            if (t_from is not None and t < t_from) or (t_to is not None and t > t_to):
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def recorded_traffic(key: str):
    """DRAM bytes per launch of an ncu capture, recorded in profiles/traffic.json under key,
    or None when the kernel source has changed since the capture (its sha256 prefix
    differs) or nothing is recorded."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[key]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("source_sha256_16") != sha or rec.get("dram_bytes_per_launch") is None:
        return None
    return int(rec["dram_bytes_per_launch"])


def prefill_bytes(wl, lengths, o_bytes=None) -> int:
    """Algorithmic bytes of one chunk-forward: every input read once, o and S_T written once
    (S0 read once when given); q and k are counted once per query/key head (value heads in a
    group share them). o_bytes is the size of one output element: by default that of the
    input dtype, the algorithmic count (2048 B per token and head for bf16 inputs, d = 128);
    the kernel writes o in fp32 (o_bytes = 4, 2304 B)."""
    es = torch.finfo(wl.dtype).bits // 8
    ob = es if o_bytes is None else o_bytes
    T = int(sum(lengths))
    # q, k per query/key head; v, w, b per value head; log_alpha fp32; o
    per_token = (wl.h_qk * 2 * wl.dk * es
                 + wl.h_v * (2 * wl.dv * es + wl.dk * es + 4 * wl.dk + ob * wl.dv))
    state = wl.n_seq * wl.h_v * wl.dk * wl.dv * 4
    return T * per_token + state * (2 if wl.S0_std else 1)


def hbm_roofline(nbytes: int, nbytes_f32o: int, ms: float, hbm: float, peak_src: str, traffic, **extra):
    """The HBM roofline of one chunk-forward launch of ms milliseconds: achieved = the
    algorithmic bytes / time; the same with o counted as the fp32 it is written in
    alongside."""
    ach = nbytes / (ms / 1000.0) / 1e9
    ach32 = nbytes_f32o / (ms / 1000.0) / 1e9
    r = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "traffic": traffic,
         "peak_source": f"{peak_src} hbm_gbs", "algorithmic_bytes_per_launch": nbytes,
         "fp32_o": {"achieved": ach32, "frac": ach32 / hbm, "algorithmic_bytes_per_launch": nbytes_f32o}}
    r.update(extra)
    return r


def prologue_bytes(wl, lengths) -> int:
    """Algorithmic bytes of one chunk-forward with the fused pre-processing: the raw
    projections (all in the input dtype, the decay pre-activation included) read once, o
    (fp32) and S_T written once."""
    es = torch.finfo(wl.dtype).bits // 8
    T = int(sum(lengths))
    per_token = wl.h_qk * 2 * wl.dk * es + wl.h_v * (2 * wl.dv * es + 2 * wl.dk * es + 4 * wl.dv)
    state = wl.n_seq * wl.h_v * wl.dk * wl.dv * 4
    return T * per_token + state * (2 if wl.S0_std else 1)


def backward_bytes(wl, lengths) -> int:
    """Algorithmic bytes of one backward: the forward's inputs and dO read once, every
    gradient (fp32) written once, S0 read and dS0 written."""
    es = torch.finfo(wl.dtype).bits // 8
    T = int(sum(lengths))
    reads = wl.h_qk * 2 * wl.dk * es + wl.h_v * (2 * wl.dv * es + wl.dk * es + 4 * wl.dk + 4 * wl.dv)
    writes = wl.h_qk * 2 * wl.dk * 4 + wl.h_v * (2 * wl.dv * 4 + 2 * wl.dk * 4)
    state = wl.n_seq * wl.h_v * wl.dk * wl.dv * 4
    return T * (reads + writes) + state * 2


def backward_flops(wl, lengths) -> int:
    """Algorithmic fp32 flops of one backward by the per-token adjoint: per token, value
    head and state element, 7 to regenerate S_prev (r: one FMA; update: a multiply and two
    FMAs) and 21 for the adjoint (ten FMAs: dS += q dO, r, dx, dr, dS', de, dk (two),
    dalpha, dq; one multiply: dS <- alpha dS'). The kernel's second forward pass (the
    recompute from checkpoints) is not counted."""
    return int(sum(lengths)) * wl.h_v * wl.dk * wl.dv * 28


def serving_bytes(wl, n_tok: int) -> int:
    """Algorithmic bytes of one serving-decode step: each active state read and written
    once, plus n_tok tokens of input and output per sequence."""
    es = torch.finfo(wl.dtype).bits // 8
    n = wl.n_seq
    io = n * n_tok * (wl.h_qk * 2 * wl.dk * es + wl.h_v * (2 * wl.dv * es + wl.dk * es + 4 * wl.dk + 4 * wl.dv))
    return io + 2 * n * wl.h_v * wl.dk * wl.dv * 4


def decode_bytes(wl) -> int:
    es = torch.finfo(wl.dtype).bits // 8
    n = wl.n_seq
    io = n * (wl.h_qk * 2 * wl.dk * es + wl.h_v * (2 * wl.dv * es + wl.dk * es + 4 * wl.dk + 4 * wl.dv))
    return io + 2 * n * wl.h_v * wl.dk * wl.dv * 4


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_baseline(seconds_target: float = 10.0):
    """The oracle as it stands on the prefill workload's whole batch (8 x 4096 tokens, 16
    heads), repeated until about seconds_target of CPU time has been spent."""
    import oracle
    from gated_delta_rule_160_b200 import workloads as W
    wl = W.WORKLOADS[PREFILL]
    d = W.prefill_inputs(wl, "cpu")
    args = [d[k] for k in ("q", "k", "v", "log_alpha", "b", "w")]
    threads = oracle.max_threads()
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.fwd_ref(*args, n_seq=wl.n_seq, want_state=False)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= seconds_target or reps >= 50:
            break
    tokens = reps * sum(d["lengths"])
    return {"value": tokens / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"the whole {PREFILL} batch ({wl.n_seq} x {wl.T} tokens, {wl.h_v} heads), "
                      f"{reps} pass(es), fp64 oracle, {dt:.1f} s"}


def run_reference(args, world, rank):
    """Reference arm: the oracle on this host's cores. A step is one bounded sample of the
    prefill workload: sequence 0, all 16 heads, 4096 tokens."""
    if rank != 0:
        return
    import oracle
    from gated_delta_rule_160_b200 import workloads as W
    wl = W.WORKLOADS[PREFILL]
    d = W.prefill_inputs(wl, "cpu", n_seq=1)
    run = lambda: oracle.fwd_ref(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], want_state=False)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    val = wl.T * args.steps / dt
    sample = f"sequence 0 of {PREFILL} ({wl.T} tokens, all {wl.h_v} heads) per step"
    print(json.dumps({
        "impl": "reference", "metric": "GDN-2 chunk-fwd tokens/s", "value": val, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": PREFILL, "sample": sample},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": oracle.max_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    if not torch.cuda.is_available():
        raise SystemExit("libgdn2 needs a CUDA device")
    import gated_delta_rule_160_b200 as G
    from gated_delta_rule_160_b200 import workloads as W

    G.load_library()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    hbm, peak_src = peaks()

    # ---------------- prefill (headline)
    wl = W.WORKLOADS[PREFILL]
    d = W.prefill_inputs(wl, dev)
    tokens_per_step = int(sum(d["lengths"]))
    o = torch.empty(d["v"].shape, dtype=torch.float32, device=dev)
    S_T = torch.empty((wl.n_seq, wl.h_v, wl.dk, wl.dv), dtype=torch.float32, device=dev)
    step = lambda: G.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=d["S0"],
                                    n_seq=d["n_seq"], o=o, S_T=S_T, stream=stream)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t_begin = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_begin.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms_local = t_begin.elapsed_time(t_end) / args.steps
    ms = max_over_ranks(ms_local, world)
    kern_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    value = world * tokens_per_step / (ms / 1000.0)
    roofline = hbm_roofline(prefill_bytes(wl, d["lengths"]), prefill_bytes(wl, d["lengths"], 4), kern_ms, hbm,
                            peak_src, recorded_traffic("chunk_tc_prefill_b8_h16_t4096"),
                            kernel="gdn2 chunk-forward", kernel_ms=kern_ms)

    o_device_run = o.cpu()  # the timed prefill's output, checked against the end-to-end path below

    # The SM clock under sustained load of the same kernel: the timed region above lasts
    # milliseconds, shorter than nvidia-smi's 50 ms sampling, so its record mostly sees the
    # GPU idle around it. Here the step runs back to back for half a second and only the
    # samples that arrive meanwhile count. (Not part of any timed figure.)
    with ClockSampler(local) as loaded:
        l_from = time.perf_counter()
        while time.perf_counter() - l_from < 0.5:
            for _ in range(40):
                step()
            torch.cuda.synchronize()
        l_to = time.perf_counter()
    clocks_loaded = loaded.summary(l_from + 0.06, l_to)

    # ---------------- prefill with the fused pre-processing (raw projections in)
    gen = torch.Generator(device=dev).manual_seed(wl.seed + 17)
    T_all = tokens_per_step
    rn = lambda *shp: torch.randn(*shp, generator=gen, device=dev).to(wl.dtype)
    raw = dict(q=rn(T_all, wl.h_qk, wl.dk), k=rn(T_all, wl.h_qk, wl.dk), a=rn(T_all, wl.h_v, wl.dk),
               b=rn(T_all, wl.h_v, wl.dk), w=rn(T_all, wl.h_v, wl.dv))
    pstep = lambda: G.gdn2_chunk_fwd(raw["q"], raw["k"], d["v"], raw["a"], raw["b"], raw["w"], S0=d["S0"],
                                     n_seq=d["n_seq"], o=o, S_T=S_T, stream=stream, prologue=True)
    for _ in range(3):
        pstep()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(PROLOGUE_TIMED_STEPS):
        pstep()
    e1.record(stream)
    torch.cuda.synchronize()
    pms = max_over_ranks(e0.elapsed_time(e1) / PROLOGUE_TIMED_STEPS, world)

    # For comparison only: the same pre-processing left to the caller as torch elementwise
    # ops, then the plain kernel on the activated inputs.
    def ustep():
        with torch.cuda.stream(stream):
            nf = torch.nn.functional
            qn = nf.normalize(raw["q"].float(), dim=-1, eps=1e-12).to(wl.dtype)
            kn = nf.normalize(raw["k"].float(), dim=-1, eps=1e-12).to(wl.dtype)
            la = nf.softplus(raw["a"].float()).neg_()
            bs = torch.sigmoid(raw["b"].float()).to(wl.dtype)
            ws = torch.sigmoid(raw["w"].float()).to(wl.dtype)
        G.gdn2_chunk_fwd(qn, kn, d["v"], la, bs, ws, S0=d["S0"], n_seq=d["n_seq"], o=o, S_T=S_T, stream=stream)
    for _ in range(3):
        ustep()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(PROLOGUE_TIMED_STEPS):
        ustep()
    e1.record(stream)
    torch.cuda.synchronize()
    ums = max_over_ranks(e0.elapsed_time(e1) / PROLOGUE_TIMED_STEPS, world)

    pbytes = prologue_bytes(wl, d["lengths"])
    pach = pbytes / (pms / 1000.0) / 1e9
    prologue = {"metric": "GDN-2 chunk-fwd tokens/s, fused pre-processing", "value": world * T_all / (pms / 1000.0),
                "unit": "tokens/s", "ms_per_step": pms, "steps": PROLOGUE_TIMED_STEPS,
                "config": {"workload": f"{PREFILL} from raw projections (bf16 decay pre-activation)"},
                "roofline": {"bound": "hbm", "achieved": pach, "peak": hbm, "unit": "GB/s", "frac": pach / hbm,
                             "traffic": recorded_traffic("chunk_tc_prologue_prefill_b8_h16_t4096"),
                             "peak_source": f"{peak_src} hbm_gbs", "algorithmic_bytes_per_launch": pbytes},
                "unfused_ms_per_step": ums,
                "unfused": "the same pre-processing as torch elementwise ops, then gdn2_chunk_fwd (comparison)"}
    del raw

    # ---------------- backward (gradients of sum(o * dO)), same workload
    dO_b = torch.randn(o.shape, generator=torch.Generator(device=dev).manual_seed(wl.seed + 29), device=dev)
    sh_b = G.make_shape(d["q"], d["v"], d["n_seq"], torch.float32)
    ws_b = torch.empty(int(G.load_library().gdn2_chunk_bwd_workspace_size(ctypes.byref(sh_b))),
                       dtype=torch.uint8, device=dev)
    bstep = lambda: G.gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], dO_b, S0=d["S0"],
                                     n_seq=d["n_seq"], workspace=ws_b, stream=stream)
    bstep()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(BACKWARD_TIMED_STEPS):
        bstep()
    e1.record(stream)
    torch.cuda.synchronize()
    bms = max_over_ranks(e0.elapsed_time(e1) / BACKWARD_TIMED_STEPS, world)
    bbytes = backward_bytes(wl, d["lengths"])
    bach = bbytes / (bms / 1000.0) / 1e9
    bflops = backward_flops(wl, d["lengths"])
    btf = bflops / (bms / 1000.0) / 1e12
    backward = {"metric": "GDN-2 backward tokens/s", "value": world * T_all / (bms / 1000.0), "unit": "tokens/s",
                "ms_per_step": bms, "steps": BACKWARD_TIMED_STEPS,
                "config": {"workload": f"{PREFILL}, gradients of sum(o * dO) (per-token adjoint, fp32, 8 value columns per warp)"},
                "roofline": {"bound": "alu", "achieved": btf, "peak": FP32_SIMT_TFLOPS, "unit": "TFLOP/s",
                             "frac": btf / FP32_SIMT_TFLOPS, "traffic": None,
                             "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flop x 1965 MHz",
                             "algorithmic_flops_per_launch": bflops,
                             "hbm": {"achieved": bach, "peak": hbm, "unit": "GB/s", "frac": bach / hbm,
                                     "algorithmic_bytes_per_launch": bbytes,
                                     "traffic": recorded_traffic("chunk_bwd_prefill_b8_h16_t4096")}}}
    del dO_b, ws_b

    # ---------------- grouped heads: 16 query/key heads shared by 32 value heads, with S0
    gwl = W.WORKLOADS[GROUPED]
    gd = W.prefill_inputs(gwl, dev)
    g_o = torch.empty(gd["v"].shape, dtype=torch.float32, device=dev)
    g_S = torch.empty_like(gd["S0"])
    gstep = lambda: G.gdn2_chunk_fwd(gd["q"], gd["k"], gd["v"], gd["log_alpha"], gd["b"], gd["w"], S0=gd["S0"],
                                     n_seq=gd["n_seq"], o=g_o, S_T=g_S, stream=stream)
    for _ in range(3):
        gstep()
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for _ in range(GROUPED_TIMED_STEPS):
        gstep()
    e1.record(stream)
    torch.cuda.synchronize()
    gms = max_over_ranks(e0.elapsed_time(e1) / GROUPED_TIMED_STEPS, world)
    g_T = int(sum(gd["lengths"]))
    grouped = {"metric": "GDN-2 chunk-fwd tokens/s, grouped heads", "value": world * g_T / (gms / 1000.0),
               "unit": "tokens/s", "ms_per_step": gms, "steps": GROUPED_TIMED_STEPS,
               "config": {"workload": GROUPED, "global_batch": gwl.n_seq, "seq_len": gwl.T, "qk_heads": gwl.h_qk,
                          "v_heads": gwl.h_v, "dk": gwl.dk, "dv": gwl.dv,
                          "bytes": "q, k counted once per query/key head"},
               "roofline": hbm_roofline(prefill_bytes(gwl, gd["lengths"]), prefill_bytes(gwl, gd["lengths"], 4), gms,
                                        hbm, peak_src, recorded_traffic("chunk_tc_grouped_b2_qk16_v32"))}
    del gd, g_o, g_S

    # ---------------- packed sequences of mixed lengths (cu_seqlens), longest first
    vwl = W.WORKLOADS[VARLEN]
    vd = W.prefill_inputs(vwl, dev)
    all_lengths = list(vd["lengths"])
    if world > 1:
        # one batch split across the ranks (data parallel, no exchange): each rank keeps the
        # sequences the longest-processing-time-first shard gives it, packed anew
        from gated_delta_rule_160_b200.sharding import pack, shard_sequences
        mine = shard_sequences(all_lengths, world, rank)
        ranges, cu = pack(all_lengths, mine)
        idx = torch.cat([torch.arange(a, z, device=dev) for a, z in ranges]) if ranges else \
            torch.zeros(0, dtype=torch.long, device=dev)
        for k in ("q", "k", "v", "log_alpha", "b", "w"):
            vd[k] = vd[k].index_select(0, idx).contiguous()
        vd["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=dev)
        vd["lengths"] = [all_lengths[i] for i in mine]
    v_o = torch.empty(vd["v"].shape, dtype=torch.float32, device=dev)
    v_S = torch.empty((len(vd["lengths"]), vwl.h_v, vwl.dk, vwl.dv), dtype=torch.float32, device=dev)
    sh_v = G.make_shape(vd["q"], vd["v"], len(vd["lengths"]), torch.float32)
    ws_v = torch.empty(max(1, G.gdn2_chunk_fwd_workspace_size(sh_v, True)), dtype=torch.uint8, device=dev)
    vstep = lambda: G.gdn2_chunk_fwd(vd["q"], vd["k"], vd["v"], vd["log_alpha"], vd["b"], vd["w"],
                                     cu_seqlens=vd["cu_seqlens"], o=v_o, S_T=v_S, workspace=ws_v, stream=stream)
    for _ in range(3):
        vstep()
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for _ in range(VARLEN_TIMED_STEPS):
        vstep()
    e1.record(stream)
    torch.cuda.synchronize()
    vms = max_over_ranks(e0.elapsed_time(e1) / VARLEN_TIMED_STEPS, world)
    v_T = int(sum(all_lengths))  # the whole batch, over all ranks
    varlen = {"metric": "GDN-2 chunk-fwd tokens/s, packed mixed lengths", "value": v_T / (vms / 1000.0),
              "unit": "tokens/s", "ms_per_step": vms, "steps": VARLEN_TIMED_STEPS,
              "scaling": "strong" if world > 1 else "n/a",
              "config": {"workload": VARLEN, "sequences": len(all_lengths), "tokens": v_T,
                         "lengths": f"{min(all_lengths)}..{max(all_lengths)}", "heads": vwl.h_v,
                         "dk": vwl.dk, "dv": vwl.dv,
                         "parallelism": f"sequences sharded over {world} ranks (longest first)" if world > 1
                         else "one GPU"},
              "roofline": hbm_roofline(prefill_bytes(vwl, vd["lengths"]), prefill_bytes(vwl, vd["lengths"], 4), vms,
                                       hbm, peak_src, None)}
    del vd, v_o, v_S, ws_v

    # ---------------- decode (the second metric)
    dwl = W.WORKLOADS[DECODE]
    S = W.decode_state(dwl, dev)
    dec_in = [W.decode_inputs(dwl, s, dev) for s in range(8)]
    do = torch.empty(dec_in[0]["v"].shape, dtype=torch.float32, device=dev)
    dstep = lambda i: G.gdn2_decode_step(*(dec_in[i % 8][k] for k in ("q", "k", "v", "log_alpha", "b", "w")),
                                         S, o=do, stream=stream)
    for i in range(5):
        dstep(i)
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for i in range(DECODE_TIMED_STEPS):
        dstep(i)
    e1.record(stream)
    torch.cuda.synchronize()
    dms = max_over_ranks(e0.elapsed_time(e1) / DECODE_TIMED_STEPS, world)
    dbytes = decode_bytes(dwl)
    dach = dbytes / (dms / 1000.0) / 1e9
    decode = {"metric": "GDN-2 decode tokens/s", "value": world * dwl.n_seq / (dms / 1000.0),
              "unit": "tokens/s", "ms_per_step": dms, "steps": DECODE_TIMED_STEPS,
              "config": {"workload": DECODE, "n_seq": dwl.n_seq, "heads": dwl.h_v, "dk": dwl.dk,
                         "dv": dwl.dv, "state_bytes": dwl.n_seq * dwl.h_v * dwl.dk * dwl.dv * 4},
              "roofline": {"bound": "hbm", "achieved": dach, "peak": hbm, "unit": "GB/s",
                           "frac": dach / hbm,
                           "traffic": recorded_traffic("decode_256seq_h32"),
                           "peak_source": f"{peak_src} hbm_gbs",
                           "algorithmic_bytes_per_launch": dbytes}}
    del S, dec_in

    # ---------------- serving decode: states in a slot pool, SERVING_TOKENS per step
    pool = torch.zeros((2 * dwl.n_seq, dwl.h_v, dwl.dk, dwl.dv), dtype=torch.float32, device=dev)
    perm = torch.randperm(2 * dwl.n_seq, generator=torch.Generator().manual_seed(dwl.seed))[:dwl.n_seq]
    pool[perm.to(dev)] = W.decode_state(dwl, dev)
    slots = perm.to(torch.int32).to(dev)
    srv_in = []
    for s_ in range(2):
        t_ = W.token_inputs(dwl.n_seq * SERVING_TOKENS, dwl.h_qk, dwl.h_v, dwl.dk, dwl.dv, dwl.dtype, dev,
                            dwl.seed * 7919 + s_)
        srv_in.append({k: t.view(dwl.n_seq, SERVING_TOKENS, *t.shape[1:]) for k, t in t_.items()})
    so = torch.empty((dwl.n_seq, SERVING_TOKENS, dwl.h_v, dwl.dv), dtype=torch.float32, device=dev)
    sstep = lambda i: G.gdn2_decode_multi(*(srv_in[i % 2][k] for k in ("q", "k", "v", "log_alpha", "b", "w")),
                                          pool, slots=slots, o=so, stream=stream)
    for i in range(5):
        sstep(i)
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for i in range(SERVING_TIMED_STEPS):
        sstep(i)
    e1.record(stream)
    torch.cuda.synchronize()
    sms = max_over_ranks(e0.elapsed_time(e1) / SERVING_TIMED_STEPS, world)
    sbytes = serving_bytes(dwl, SERVING_TOKENS)
    sach = sbytes / (sms / 1000.0) / 1e9
    serving = {"metric": "GDN-2 serving decode tokens/s",
               "value": world * dwl.n_seq * SERVING_TOKENS / (sms / 1000.0), "unit": "tokens/s",
               "ms_per_step": sms, "steps": SERVING_TIMED_STEPS,
               "config": {"workload": f"{DECODE}, states at seeded-random slots of a {2 * dwl.n_seq}-state "
                                      f"pool, {SERVING_TOKENS} tokens per sequence and step",
                          "n_seq": dwl.n_seq, "heads": dwl.h_v, "n_tok": SERVING_TOKENS,
                          "pool_slots": 2 * dwl.n_seq},
               "roofline": {"bound": "hbm", "achieved": sach, "peak": hbm, "unit": "GB/s", "frac": sach / hbm,
                            "traffic": recorded_traffic("decode_multi_serving_256seq_h32"),
                            "peak_source": f"{peak_src} hbm_gbs",
                            "algorithmic_bytes_per_launch": sbytes}}
    del pool, srv_in, so

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        names = ("q", "k", "v", "log_alpha", "b", "w")
        host = {k: d[k].cpu().pin_memory() for k in names}
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o_host.numel() * o_host.element_size()
        dev_in = {k: torch.empty_like(d[k]) for k in names}
        del d

        # Sequence by sequence: inputs go up on `up`, the prefill runs on `stream`, o comes
        # down on `down`, so the copies of one sequence overlap the others' work (the link is
        # full duplex). Every sequence is one gdn2_chunk_fwd call on its slice of the batch.
        # Consecutive steps overlap as a stream of batches would: a sequence's upload waits
        # only for the previous step's prefill of that sequence (which read the device
        # buffers it overwrites), its prefill for the previous step's download of its o.
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(wl.n_seq)]
        ev_out = [torch.cuda.Event() for _ in range(wl.n_seq)]
        ev_dl = [torch.cuda.Event() for _ in range(wl.n_seq)]

        def e2e_step():
            for s_ in range(wl.n_seq):
                sl = slice(s_ * wl.T, (s_ + 1) * wl.T)
                up.wait_event(ev_out[s_])
                with torch.cuda.stream(up):
                    for k in names:
                        dev_in[k][sl].copy_(host[k][sl], non_blocking=True)
                    ev_in[s_].record(up)
                stream.wait_event(ev_in[s_])
                stream.wait_event(ev_dl[s_])
                G.gdn2_chunk_fwd(*(dev_in[k][sl] for k in names), n_seq=1, o=o[sl], S_T=S_T[s_:s_ + 1],
                                 stream=stream)
                ev_out[s_].record(stream)
                down.wait_event(ev_out[s_])
                with torch.cuda.stream(down):
                    o_host[sl].copy_(o[sl], non_blocking=True)
                    ev_dl[s_].record(down)

        for _ in range(2):
            e2e_step()
        stream.wait_stream(down)
        torch.cuda.synchronize()
        n_e2e = max(3, min(args.steps, 10))
        barrier(world)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        up.wait_stream(stream)  # no upload of the timed steps starts before a
        for _ in range(n_e2e):
            e2e_step()
        stream.wait_stream(down)  # b after every step's last download
        b_.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(a.elapsed_time(b_) / n_e2e, world)
        e2e = {"value": world * tokens_per_step / (ems / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems,
               "steps": n_e2e,
               "pipeline": "per sequence: upload, prefill and download on three streams; consecutive steps overlap",
               "o_equals_device_run": bool(torch.equal(o_host, o_device_run))}
    del o_device_run

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline()

    if rank == 0:
        # the two headline metrics come first and last: the driver keeps the standard keys
        # and the last 1500 characters of the line, so decode sits at its end
        line = {
            "metric": "GDN-2 chunk-fwd tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": PREFILL, "global_batch": wl.n_seq * world, "seq_len": wl.T,
                       "heads": wl.h_v, "dk": wl.dk, "dv": wl.dv, "parallelism": f"replicas{world}",
                       "inputs": "bf16 q,k,v,b,w; fp32 log_alpha, state and output",
                       "l2": "inputs (1.07 GB per rank) larger than L2; no flush"},
            "roofline": roofline,
            "e2e": e2e,
            "grouped": grouped,
            "varlen": varlen,
            "prefill_prologue": prologue,
            "backward": backward,
            "serving_decode": serving,
            "cpu_baseline": base,
            "decode": decode,
            "clocks": clocks.summary(),
            "clocks_loaded": clocks_loaded,
            "gpu_launches": args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
