#!/usr/bin/env python
"""Benchmark of the fused MoE expert-FFN forward on B200.

One step = the whole hot path on one batch: the routing planner (moe_align)
followed by the fused forward (gate/up GEMM + SwiGLU, down GEMM, top-k
weighted reduction) through the C ABI.  Default workload: the bf16 decode
regime K=4096, N=4096 (intermediate 2048), E=256, top-6, T=256 tokens
(block_m 128).  Inputs are synthetic and seeded (``workloads``); they are
uploaded before the timed region.  The expert weights (12.9 GB) are larger
than L2, so every step streams them from HBM.

Printed (rank 0, one JSON line): the metric's value in TFLOP/s of routed
FLOPs (3*T*top_k*K*N per call) for the whole job, microseconds per call,
effective weight GB/s, the roofline of the dominant kernel (the gate/up
phase, timed with CUDA events recorded by the library on the launching
stream), the end-to-end figure through host buffers, SM clocks sampled during
the timed region, and the CPU oracle timed on a bounded token sample.

Other rows: ``--workload C3F4`` / ``C4F4`` run the MXFP4-weight path; ``--router`` starts each step
from router logits (``moe_route_align``); ``--router --shared S`` adds S shared experts.

Multi-GPU: ``torchrun --nproc-per-node N bench.py --gpus N``; every rank is an
independent replica with all experts resident (no collective on the data
path); time is the max over ranks, ``value`` the sum of all ranks' work.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "fused MoE fwd µs/call + TFLOP/s (% of roofline) at tokens 64–8192, 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default="C2", choices=W.workload_names())
    ap.add_argument("--tokens", type=int, default=256)
    ap.add_argument("--experts", type=int, default=0, help="override the workload's expert count (profiling)")
    ap.add_argument("--seed", type=int, default=W.DEFAULT_SEED)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the CPU oracle baseline")
    ap.add_argument("--cpu-threads", type=int, default=0,
                    help="threads of the CPU oracle (baseline and reference arm); 0 = every host core")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--router", action="store_true",
                    help="start each step from router logits (moe_route_align) instead of routed ids")
    ap.add_argument("--shared", type=int, default=0,
                    help="shared experts after the routed ones (every token, weight 1); needs --router")
    ap.add_argument("--stages", type=int, default=0)
    ap.add_argument("--ctas", type=int, default=0)
    ap.add_argument("--flush-l2", action="store_true",
                    help="flush L2 between steps (automatic when the touched weights are < 4x L2)")
    args = ap.parse_args(argv)
    if args.shared and not args.router:
        ap.error("--shared needs --router (the router appends the shared experts' routes)")
    if args.shared < 0:
        ap.error("--shared must be >= 0")
    if args.cpu_threads < 0:
        ap.error("--cpu-threads must be >= 0")
    return args


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def cost_model(sh: W.Shape, topk_ids: np.ndarray, peaks: dict):
    """Routed FLOPs, touched weight bytes and the path roofline time (s)."""
    R = sh.T * sh.top_k
    flops = 3.0 * R * sh.K * sh.N
    counts = np.bincount(topk_ids.reshape(-1)[(topk_ids.reshape(-1) >= 0) & (topk_ids.reshape(-1) < sh.E)],
                         minlength=sh.E)
    touched = int((counts > 0).sum())
    # weight bytes per value: bf16 2; mxfp8 1 + 1/32 (e8m0 per 32); MXFP4 1/2 + 1/32
    b = {"bf16": 2.0, "mxfp8": 1.0 + 1.0 / 32.0, "mxfp4": 0.5 + 1.0 / 32.0}[sh.dtype]
    bytes_w = touched * 1.5 * sh.N * sh.K * b
    p_tc = peaks["bf16_tflops"] * (1.0 if sh.dtype == "bf16" else 2.0) * 1e12
    bw = peaks["hbm_gbs"] * 1e9
    t_flop, t_hbm = flops / p_tc, bytes_w / bw
    # gate/up phase: w1 of the touched experts, the routed rows of x, the intermediate written once
    bx = 2.0 if sh.dtype == "bf16" else 1.0 + 1.0 / 32.0
    p1_bytes = touched * sh.N * sh.K * b + R * sh.K * bx + R * sh.I * bx
    p1_flops = 2.0 * R * sh.K * sh.N
    # the whole path's algorithmic HBM bytes: touched weights, x (+ its scales) read once, out written
    # once, the routing read, the planner's arrays written (sorted ids, expert ids, the padded total)
    cap = R + sh.E * (sh.block_m - 1)
    full = {"weights": bytes_w, "x": sh.T * sh.K * bx, "out": 2.0 * sh.T * sh.K, "routing": 8.0 * R,
            "plan": 4.0 * cap + 4.0 * ((cap + sh.block_m - 1) // sh.block_m) + 4.0}
    return dict(R=R, flops=flops, touched=touched, bytes_w=bytes_w, t_flop=t_flop, t_hbm=t_hbm,
                t_roof=max(t_flop, t_hbm), bound="tensor" if t_flop > t_hbm else "hbm", p_tc=p_tc, bw=bw,
                p1_bytes=p1_bytes, p1_flops=p1_flops, bytes_full=sum(full.values()), bytes_parts=full)


class ClockSampler:
    """nvidia-smi SM clocks / throttle reasons sampled every 100 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return self.summary()

    def summary(self):
        sm, mx, reasons, watts = [], None, set(), []
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
            try:
                watts.append(float(f[3]))
            except ValueError:
                pass
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w": statistics.median(watts) if watts else None}


def kernel_traffic(kernel: str, workload_tag: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (its sha256 is recorded in the summary)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload_tag}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    if not m or not h:
        return None
    src = os.path.join(ROOT, "mixture_experts_ffn_planner_b200", "csrc", "fused_moe.cu")
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != h.group(1):
        return None
    return float(m.group(1))


# ----------------------------------------------------------------------------- CPU oracle legs
def oracle_threads(requested: int) -> int:
    return requested if requested > 0 else (os.cpu_count() or 1)


def oracle_sample_rate(sh: W.Shape, inp: dict, seconds: float, seed: int, threads: int = 0):
    """Times the oracle on a growing token sample until ~`seconds` of work; returns
    (TFLOP/s, threads, description)."""
    thr = oracle_threads(threads)
    n, spent, flops = 1, 0.0, 0.0
    perm = np.random.default_rng(seed).permutation(sh.T)
    used = 0
    while spent < seconds and used < sh.T:
        toks = np.sort(perm[used:used + n]).astype(np.int32)
        t0 = time.perf_counter()
        _run_oracle(sh, inp, toks, thr)
        dt = time.perf_counter() - t0
        spent += dt
        flops += 3.0 * len(toks) * sh.top_k * sh.K * sh.N
        used += len(toks)
        n = max(1, min(sh.T - used, int(n * max(1.0, min(4.0, (seconds - spent) / max(dt, 1e-3))))))
    desc = f"{used} of {sh.T} tokens ({used * sh.top_k} routes) of {sh.name} T={sh.T}, oracle in float64"
    return flops / spent / 1e12, thr, desc, spent


def _run_oracle(sh, inp, toks, thr):
    import oracle

    if sh.dtype == "bf16":
        return oracle.fused_moe_bf16(inp["x"], inp["w1"], inp["w2"], inp["topk_ids"], inp["topk_weights"],
                                     tokens=toks, nthreads=thr)
    fwd = oracle.fused_moe_mxfp4 if sh.dtype == "mxfp4" else oracle.fused_moe_mxfp8
    return fwd(inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], inp["w2"], inp["w2_scales"],
               inp["topk_ids"], inp["topk_weights"], tokens=toks, nthreads=thr)


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sh = W.shape(args.workload, args.tokens, **({"E": args.experts} if args.experts else {}))
    inp = W.inputs(sh, seed=args.seed)
    thr = oracle_threads(args.cpu_threads)
    # calibrate: tokens per step such that all steps fit in ~2 minutes
    t0 = time.perf_counter()
    _run_oracle(sh, inp, np.array([0], np.int32), thr)
    per_tok = max(time.perf_counter() - t0, 1e-4)
    budget = 120.0 / max(1, args.steps + args.warmup)
    ntok = int(max(1, min(sh.T, budget / per_tok)))
    perm = np.random.default_rng(args.seed).permutation(sh.T)
    times = []
    for i in range(args.warmup + args.steps):
        toks = np.sort(np.roll(perm, -i * ntok)[:ntok]).astype(np.int32)
        t0 = time.perf_counter()
        _run_oracle(sh, inp, toks, thr)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    flops = 3.0 * ntok * sh.top_k * sh.K * sh.N * len(times)
    value = flops / total / 1e12
    sample = f"{ntok} of {sh.T} tokens per step ({ntok * sh.top_k} routes) of {sh.name} T={sh.T}"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded workloads generator)",
            "config": {"workload": f"{sh.name}: {sh.dtype} K={sh.K} N={sh.N} E={sh.E} top_k={sh.top_k} T={sh.T}"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
class Problem:
    """Device-resident inputs of one workload and one step of the hot path."""

    def __init__(self, sh: W.Shape, inp: dict, dev, stages: int = 0, ctas: int = 0, router: bool = False,
                 n_shared: int = 0):
        import torch

        import mixture_experts_ffn_planner_b200 as moe

        self.sh, self.inp, self.dev, self.moe = sh, inp, dev, moe

        def up(a, dtype=None):
            t = torch.from_numpy(np.ascontiguousarray(a))
            return (t.view(dtype) if dtype is not None else t).to(dev)

        bm = self.bm = sh.block_m
        self.router = router
        self.n_shared = n_shared  # shared experts after the sh.E routed ones (router path only)
        if router:
            # the step starts from router logits: moe_route_align writes ids and weights
            self.logits = up(inp["router_logits"])
            self.bias = None if inp["router_bias"] is None else up(inp["router_bias"])
            self.ids = torch.empty((sh.T, sh.top_k + n_shared), dtype=torch.int32, device=dev)
            self.tw = torch.empty((sh.T, sh.top_k + n_shared), dtype=torch.float32, device=dev)
        else:
            self.ids, self.tw = up(inp["topk_ids"]), up(inp["topk_weights"])
        cap = moe.moe_align_capacity(sh.T, sh.top_k + n_shared, sh.E + n_shared, bm)
        self.s_ids = torch.empty(cap, dtype=torch.int32, device=dev)
        self.e_ids = torch.empty((cap + bm - 1) // bm, dtype=torch.int32, device=dev)
        self.ntpp = torch.empty(1, dtype=torch.int32, device=dev)
        self.out = torch.empty((sh.T, sh.K), dtype=torch.bfloat16, device=dev)
        if sh.dtype == "bf16":
            self.x = up(inp["x"], torch.bfloat16)
            self.w1, self.w2 = up(inp["w1"], torch.bfloat16), up(inp["w2"], torch.bfloat16)
            self.xs = self.s1 = self.s2 = None
            dt = moe.DTYPE_BF16
        else:
            self.x, self.xs, self.w1, self.w2 = up(inp["x"]), up(inp["x_scales"]), up(inp["w1"]), up(inp["w2"])
            self.s1 = moe.pack_scales_blocked(up(inp["w1_scales"]))
            self.s2 = moe.pack_scales_blocked(up(inp["w2_scales"]))
            dt = moe.DTYPE_MXFP4 if sh.dtype == "mxfp4" else moe.DTYPE_MXFP8
        self.ws = torch.empty(moe.moe_workspace_bytes(dt, sh.T, sh.K, sh.N, sh.E + n_shared, sh.top_k + n_shared, bm),
                              dtype=torch.uint8, device=dev)
        self.plain = moe.Tuning(stages, ctas, None)
        self.stages, self.ctas = stages, ctas
        # planner, gate/up phase, split-K reduction, down phase, combine (+ the router kernel for
        # batches of more than 128 tokens on the router path)
        self.launches_per_step = 5 + (1 if router and sh.T > 128 else 0)

    def fused(self, tune):
        m = self.moe
        if self.sh.dtype == "bf16":
            m.fused_moe_bf16(self.x, self.w1, self.w2, self.s_ids, self.e_ids, self.ntpp, self.tw, self.out, self.bm,
                             workspace=self.ws, tune=tune)
        else:
            fwd = m.fused_moe_mxfp4 if self.sh.dtype == "mxfp4" else m.fused_moe_mxfp8
            fwd(self.x, self.xs, self.w1, self.s1, self.w2, self.s2, self.s_ids, self.e_ids, self.ntpp,
                self.tw, self.out, self.bm, workspace=self.ws, tune=tune)

    def step(self, tune=None, plan_event=None):
        if plan_event is not None:
            plan_event.record()
        if self.router:
            self.moe.moe_route_align(self.logits, self.sh.top_k, self.bm, self.bias, self.ids, self.tw, self.s_ids,
                                     self.e_ids, self.ntpp, n_shared=self.n_shared)
        else:
            self.moe.moe_align(self.ids, self.sh.E, self.bm, self.s_ids, self.e_ids, self.ntpp)
        self.fused(self.plain if tune is None else tune)


def measure(prob: Problem, steps: int, warmup: int, flush_l2: bool = False, barrier=None, sample_clocks=True,
            local: int = 0):
    """Device time of `steps` steps after `warmup`.

    Pass 1 (the reported time): the steps run with nothing between their
    launches, so the library's programmatic dependent launch overlaps each
    kernel's prologue with the previous kernel.  With flush_l2 every step is
    bracketed by its own events and a >L2 buffer is written between steps
    (outside the timed windows); otherwise the steps run back to back between
    one pair of events.
    Pass 2 (the per-kernel breakdown): the same steps with the library's phase
    events recorded between its launches (events between launches can keep the
    launches from overlapping, so pass 2 is used for the per-kernel times only).
    With flush_l2, pass 3 runs the steps back to back without the flush (warm
    L2), reported beside the cold time and labelled as such.
    """
    import torch

    moe = prob.moe
    stream = torch.cuda.current_stream()
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=prob.dev) if flush_l2 else None

    def flush():
        # write a buffer 4x the L2 size, then read it back: the read evicts the
        # dirty lines the write left (their write-back happens here, outside
        # the timed window) so the next step starts with a cold, clean L2
        flush_buf.fill_(1)
        flush_buf.max()

    for _ in range(max(3, warmup)):
        prob.step()
        if flush_buf is not None:
            flush()
    moe.moe_device_status()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local) if sample_clocks else None
    if clocks:
        clocks.start()
        time.sleep(0.3)

    def timed(tunes=None, pev=None, cold=flush_l2):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)] \
            if cold else None
        t0.record(stream)
        for i in range(steps):
            if s_ev:
                s_ev[i][0].record(stream)
            prob.step(None if tunes is None else tunes[i], None if pev is None else pev[i])
            if s_ev:
                s_ev[i][1].record(stream)
                flush()
        t1.record(stream)
        torch.cuda.synchronize()
        if s_ev:
            per_step.clear()
            per_step.extend(a.elapsed_time(b) for a, b in s_ev)
            return sum(per_step)
        return t0.elapsed_time(t1)

    per_step = []
    total_ms = timed()
    median_ms = float(np.median(per_step)) if per_step else None
    if barrier:
        barrier()
    clk = clocks.stop() if clocks else None
    moe.moe_device_status()
    # pass 2: per-kernel times
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    pev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    tunes = [moe.Tuning.with_events(e, prob.stages, prob.ctas) for e in ev]
    timed(tunes, pev)
    moe.moe_device_status()
    warm_ms = None
    if flush_l2:
        prob.step()  # the last flush left L2 cold; one untimed step warms it
        warm_ms = timed(cold=False) / steps
        moe.moe_device_status()
    return {"total_ms": total_ms, "ms_step": total_ms / steps, "warm_ms_step": warm_ms, "median_ms_step": median_ms,
            "plan_ms": sum(a.elapsed_time(e[0]) for a, e in zip(pev, ev)) / steps,
            "p1_ms": sum(e[0].elapsed_time(e[1]) for e in ev) / steps,
            "p2_ms": sum(e[1].elapsed_time(e[2]) for e in ev) / steps,
            "cb_ms": sum(e[2].elapsed_time(e[3]) for e in ev) / steps,
            "clocks": clk, "launches": prob.launches_per_step * steps}


def measure_e2e(prob: Problem, steps: int, barrier=None):
    """Same steps through host buffers: pinned H2D of the step's inputs (x, its
    scales, routing) and D2H of out inside the timed region."""
    import torch

    sh, inp = prob.sh, prob.inp
    stream = torch.cuda.current_stream()
    hx = torch.from_numpy(np.ascontiguousarray(inp["x"]))
    hx = hx.view(torch.bfloat16) if sh.dtype == "bf16" else hx
    if prob.router:
        host_in = [hx.pin_memory(), torch.from_numpy(inp["router_logits"]).pin_memory()]
        dev_in = [prob.x, prob.logits]
        if prob.bias is not None:
            host_in.append(torch.from_numpy(inp["router_bias"]).pin_memory())
            dev_in.append(prob.bias)
    else:
        host_in = [hx.pin_memory(), torch.from_numpy(inp["topk_ids"]).pin_memory(),
                   torch.from_numpy(inp["topk_weights"]).pin_memory()]
        dev_in = [prob.x, prob.ids, prob.tw]
    if sh.dtype != "bf16":
        host_in.append(torch.from_numpy(np.ascontiguousarray(inp["x_scales"])).pin_memory())
        dev_in.append(prob.xs)
    host_out = torch.empty((sh.T, sh.K), dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_out.numel() * host_out.element_size()

    def one():
        for h, d in zip(host_in, dev_in):
            d.copy_(h, non_blocking=True)
        prob.step()
        host_out.copy_(prob.out, non_blocking=True)

    for _ in range(3):
        one()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1), h2d, d2h


def roofline_of_p1(sh: W.Shape, cm: dict, p1_ms: float, peaks: dict, peak_src: str):
    p1_s = p1_ms * 1e-3
    tag = f"{sh.name}_T{sh.T}"
    name = "moe_p1_kernel (gather + gate/up GEMM + SwiGLU)"
    if cm["p1_flops"] / cm["p_tc"] <= cm["p1_bytes"] / cm["bw"]:
        gbs = cm["p1_bytes"] / p1_s / 1e9
        return {"kernel": name, "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"], "traffic": kernel_traffic("moe_p1_kernel", tag),
                "peak_source": f"{peak_src} hbm_gbs", "algorithmic_bytes_per_launch": cm["p1_bytes"],
                "us_per_launch": p1_ms * 1e3}
    pk = peaks["bf16_tflops"] * (1.0 if sh.dtype == "bf16" else 2.0)
    tf = cm["p1_flops"] / p1_s / 1e12
    return {"kernel": name, "bound": "tensor", "achieved": tf, "peak": pk, "unit": "TFLOP/s", "frac": tf / pk,
            "traffic": kernel_traffic("moe_p1_kernel", tag),
            "peak_source": f"{peak_src} bf16_tflops" + ("" if sh.dtype == "bf16" else " x 2 (fp8:bf16 nominal)"),
            "algorithmic_flops_per_launch": cm["p1_flops"], "us_per_launch": p1_ms * 1e3}


def result_line(sh, cm, m, world, steps, warmup, peaks, peak_src, flush_l2):
    ms_step = m["ms_step"]
    l2 = ("L2 flushed between steps (512 MB written then read back, outside the per-step events)" if flush_l2 else
          f"inputs larger than L2 (touched expert weights {cm['bytes_w'] / 1e9:.2f} GB per step)")
    return {
        "metric": METRIC, "value": whole_job_tflops(cm["flops"], world, ms_step), "unit": "TFLOP/s",
        "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": sh.dtype,
        "data": "synthetic (seeded workloads generator, random weights)",
        "config": {"workload": f"{sh.name}: {sh.dtype} MoE FFN K={sh.K} N={sh.N} (intermediate {sh.I}) "
                               f"E={sh.E} top_k={sh.top_k} T={sh.T} block_m={sh.block_m}",
                   "tokens_per_gpu": sh.T, "parallelism": f"replicas x{world}", "l2": l2},
        "us_per_call": ms_step * 1e3,
        **({"us_per_call_median": m["median_ms_step"] * 1e3} if m.get("median_ms_step") else {}),
        "weight_GBps": cm["bytes_w"] / (ms_step * 1e-3) / 1e9,
        "path_roofline": {"bound": cm["bound"], "t_roof_us": cm["t_roof"] * 1e6,
                          "frac": cm["t_roof"] / (ms_step * 1e-3), "touched_experts": cm["touched"],
                          "routed_gflop": cm["flops"] / 1e9, "touched_weight_gb": cm["bytes_w"] / 1e9,
                          "algorithmic_hbm_gb": cm["bytes_full"] / 1e9,
                          "algorithmic_hbm_parts_gb": {k: v / 1e9 for k, v in cm["bytes_parts"].items()},
                          "peaks": peak_src},
        "phase_us": {"planner": m["plan_ms"] * 1e3, "gate_up": m["p1_ms"] * 1e3, "down": m["p2_ms"] * 1e3,
                     "reduce": m["cb_ms"] * 1e3},
        "roofline": roofline_of_p1(sh, cm, m["p1_ms"], peaks, peak_src),
        "gpu_launches": m["launches"],
        "clocks": m["clocks"],
        **({"warm": {"us_per_call": m["warm_ms_step"] * 1e3,
                     "l2": "not flushed: steps back to back, so weights can stay L2-resident (not the reported value)"}}
           if m.get("warm_ms_step") else {}),
    }


def max_over_ranks(v: float, world: int, dist=None, device=None) -> float:
    """The maximum of a per-rank value over all ranks (every rank gets it)."""
    if world == 1:
        return v
    import torch

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Replicas: every rank does the same work per step; the job's rate is the
    sum of the ranks' work over the slowest rank's step time."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def run_b200(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    barrier = dist.barrier if world > 1 else None
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()

    sh = W.shape(args.workload, args.tokens, **({"E": args.experts} if args.experts else {}))
    if args.shared:
        # weights of the routed experts followed by the shared ones
        sh_w = dataclasses.replace(sh, E=sh.E + args.shared, top_k=sh.top_k + args.shared)
        inp = W.inputs(sh_w, seed=args.seed + rank)
        # the generator's routing over the routed experts, then the shared routes (cost model and
        # CPU baseline; the timed step routes from logits on the GPU)
        ids, tw = W.routing(sh, seed=args.seed + rank)
        shared_ids = np.broadcast_to(np.arange(sh.E, sh.E + args.shared, dtype=np.int32), (sh.T, args.shared))
        inp["topk_ids"] = np.ascontiguousarray(np.concatenate([ids, shared_ids], axis=1))
        inp["topk_weights"] = np.ascontiguousarray(
            np.concatenate([tw, np.ones((sh.T, args.shared), np.float32)], axis=1))
    else:
        inp = W.inputs(sh, seed=args.seed + rank)  # every replica gets its own batch
    if args.router:
        inp["router_logits"], inp["router_bias"] = W.router_logits(sh, seed=args.seed + rank)
    cm = cost_model(sh_w if args.shared else sh, inp["topk_ids"], peaks)
    prob = Problem(sh, inp, dev, args.stages, args.ctas, router=args.router, n_shared=args.shared)
    flush = args.flush_l2 or cm["bytes_w"] < 4 * 126e6
    m = measure(prob, args.steps, args.warmup, flush_l2=flush, barrier=barrier, local=local)

    m["ms_step"] = max_over_ranks(m["ms_step"], world, dist, dev)
    line = result_line(sh, cm, m, world, args.steps, args.warmup, peaks, peak_src, flush)
    if args.router:
        line["config"]["router"] = "in the step: moe_route_align (softmax, top-k, renormalise) from fp32 logits"
    if args.shared:
        line["config"]["shared_experts"] = args.shared
    if not args.no_e2e:
        ems, h2d, d2h = measure_e2e(prob, args.steps, barrier)
        ems = max_over_ranks(ems, world, dist, dev)
        line["e2e"] = {"value": whole_job_tflops(cm["flops"], world, ems / args.steps), "unit": "TFLOP/s",
                       "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                       "us_per_call": 1e3 * ems / args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, thr, desc, spent = oracle_sample_rate(sh, inp, args.cpu_seconds, args.seed, args.cpu_threads)
        line["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                "sample": desc, "seconds": spent}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_b200(args)


if __name__ == "__main__":
    sys.exit(main())
