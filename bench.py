#!/usr/bin/env python
"""Benchmark of the fused MoE expert-FFN forward on B200.

One step = the whole hot path on one batch: the routing planner (moe_align)
followed by the fused forward (gate/up GEMM + SwiGLU, mxfp8 requant, down
GEMM, top-k weighted reduction) through the C ABI.  Default workload: the
largest configuration, C4 -- mxfp8, K=7168, N=6144 (intermediate 3072),
E=384, top-6, T=8192 tokens (block_m 128).  Inputs are synthetic and seeded
(``workloads``); they are on the device before the timed region.  The
expert weights (26 GB) are far larger than L2, so every step streams them
from HBM.

Printed (rank 0, one JSON line): the metric's value in TFLOP/s of routed
FLOPs (3*T*top_k*K*N per call) for the whole job, microseconds per call,
effective weight GB/s, the roofline of the dominant kernel (the gate/up
phase, timed with CUDA events recorded by the library on the launching
stream), the end-to-end figure through host buffers, SM clocks sampled during
the timed region, and the CPU oracle timed on a bounded token sample.

Other rows: ``--workload C3F4`` / ``C4F4`` run the MXFP4-weight path; ``--router`` starts each step
from router logits (``moe_route_align``); ``--router --shared S`` adds S shared experts.
``--sweep`` prints one such line per (configuration, token count) over every workload (one GPU).
``--peak`` measures the dense tensor-core peaks the roofline divides by (bf16 and mxfp8 GEMMs
through torch at 8192^3) and prints them as one JSON line.

Multi-GPU: ``torchrun --nproc-per-node N bench.py --gpus N``; every rank is an
independent replica with all experts resident and its own token batch (no
collective on the data path); time is the max over ranks, ``value`` the sum
of all ranks' work.  The replicas hold the same expert weights: each rank
draws E/N of the experts and the ranks all-gather them before timing.
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
    ap.add_argument("--workload", default="C4", choices=W.workload_names())
    ap.add_argument("--tokens", type=int, default=8192)
    ap.add_argument("--experts", type=int, default=0, help="override the workload's expert count (profiling)")
    ap.add_argument("--seed", type=int, default=W.DEFAULT_SEED)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the CPU oracle baseline")
    ap.add_argument("--cpu-threads", type=int, default=0,
                    help="threads of the CPU oracle (baseline and reference arm); 0 = every host core")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay figure")
    ap.add_argument("--router", action="store_true",
                    help="start each step from router logits (moe_route_align) instead of routed ids")
    ap.add_argument("--shared", type=int, default=0,
                    help="shared experts after the routed ones (every token, weight 1); needs --router")
    ap.add_argument("--stages", type=int, default=0)
    ap.add_argument("--small-batch", choices=["auto", "on", "off"], default="auto",
                    help="bf16: the library's choice between the small-batch form and the tensor-core phases "
                         "(moe_tuning.small_batch)")
    ap.add_argument("--ctas", type=int, default=0)
    ap.add_argument("--flush-l2", action="store_true",
                    help="flush L2 between steps (automatic when the touched weights are < 4x L2)")
    ap.add_argument("--sweep", action="store_true",
                    help="one line per (workload, token count) of every configuration (one GPU)")
    ap.add_argument("--sweep-workloads", default="C1,C2,C3,C4,C5,C3F4,C4F4",
                    help="comma-separated workloads of --sweep")
    ap.add_argument("--peak", action="store_true", help="measure the dense bf16 and mxfp8 tensor peaks")
    args = ap.parse_args(argv)
    if args.sweep and args.gpus != 1:
        ap.error("--sweep runs on one GPU")
    for w in args.sweep_workloads.split(","):
        if w not in W.workload_names():
            ap.error(f"--sweep-workloads: unknown workload {w}")
    if args.shared and not args.router:
        ap.error("--shared needs --router (the router appends the shared experts' routes)")
    if args.shared < 0:
        ap.error("--shared must be >= 0")
    if args.cpu_threads < 0:
        ap.error("--cpu-threads must be >= 0")
    return args


def load_peaks():
    """The roofline's denominators: HBM copy bandwidth and the dense bf16 GEMM rate from the
    measured MEASURED_PEAKS.json, and the dense mxfp8 GEMM rate from the committed
    measurement in profiles/tensor_peak_mxfp8.md (``bench.py --peak`` on a B200), else 2x the bf16
    figure (the nominal dense fp8:bf16 ratio)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        peaks, src = {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        peaks, src = dict(FALLBACK_PEAKS), "fallback"
    mx = None
    try:
        txt = open(os.path.join(ROOT, "profiles", "tensor_peak_mxfp8.md")).read()
        m = re.search(r"mxfp8_tflops_burst:\s*([0-9.]+)", txt)
        mx = float(m.group(1)) if m else None
    except OSError:
        pass
    if mx:
        peaks["mxfp8_tflops"], peaks["mxfp8_source"] = mx, "measured (profiles/tensor_peak_mxfp8.md)"
    else:
        peaks["mxfp8_tflops"], peaks["mxfp8_source"] = 2.0 * peaks["bf16_tflops"], "2 x bf16 (nominal ratio)"
    return peaks, src


def tensor_peak(sh: W.Shape, peaks: dict) -> float:
    """Dense tensor peak (TFLOP/s) of the workload's MMA kind: bf16, or mxfp8 (also for MXFP4 weights,
    which run on the same block-scaled f8f6f4 MMA)."""
    return peaks["bf16_tflops"] if sh.dtype == "bf16" else peaks.get("mxfp8_tflops", 2.0 * peaks["bf16_tflops"])


SMALL_BATCH_MODE = {"auto": 0, "on": 1, "off": -1}


def small_batch_form(sh: W.Shape, mode: int = 0) -> bool:
    """Whether fused_moe_bf16 takes its small-batch form for this shape under moe_tuning.small_batch =
    mode (the library's switch: bf16, K and N/2 multiples of 256, and by default T * top_k <= 128)."""
    ok = sh.dtype == "bf16" and sh.K % 256 == 0 and (sh.N // 2) % 256 == 0 and sh.T <= 8192
    return ok and mode >= 0 and (mode > 0 or sh.T * sh.top_k <= 128)


def cost_model(sh: W.Shape, topk_ids: np.ndarray, peaks: dict, small_batch: int = 0):
    """Routed FLOPs, touched weight bytes, the path roofline time (s) and each kernel's
    algorithmic bytes and FLOPs."""
    R = sh.T * sh.top_k
    flops = 3.0 * R * sh.K * sh.N
    flat = topk_ids.reshape(-1)
    valid = flat[(flat >= 0) & (flat < sh.E)]
    counts = np.bincount(valid, minlength=sh.E)
    touched = int((counts > 0).sum())
    Rv = int(valid.size)  # routes that reach an expert
    # weight bytes per value: bf16 2; mxfp8 1 + 1/32 (e8m0 per 32); MXFP4 1/2 + 1/32
    b = {"bf16": 2.0, "mxfp8": 1.0 + 1.0 / 32.0, "mxfp4": 0.5 + 1.0 / 32.0}[sh.dtype]
    bytes_w = touched * 1.5 * sh.N * sh.K * b
    p_tc = tensor_peak(sh, peaks) * 1e12
    bw = peaks["hbm_gbs"] * 1e9
    t_flop, t_hbm = flops / p_tc, bytes_w / bw
    # bytes per activation value: bf16 2, mxfp8 1 + 1/32; per partial-row value: fp32 / bf16
    bx = 2.0 if sh.dtype == "bf16" else 1.0 + 1.0 / 32.0
    by = 4.0 if sh.dtype == "bf16" else 2.0
    kern = {
        # gate/up: w1 of the touched experts, the routed rows of x, the intermediate written once
        "gate_up": dict(bytes=touched * sh.N * sh.K * b + Rv * sh.K * bx + Rv * sh.I * bx,
                        flops=2.0 * Rv * sh.K * sh.N, name="moe_p1_kernel (gather + gate/up GEMM + SwiGLU)",
                        ncu="moe_p1_kernel"),
        # down (+ the split-K reduction when it runs): w2, the intermediate read once, the weighted
        # partial row of every route written once (fp32 on the bf16 path, bf16 on the mxfp8 path)
        "down": dict(bytes=touched * sh.K * sh.I * b + Rv * sh.I * bx + Rv * sh.K * by,
                     flops=1.0 * Rv * sh.K * sh.N, name="moe_p2_kernel (down GEMM + routing weight)",
                     ncu="moe_p2_kernel"),
        # top-k reduction: every partial row read, out written, one flag per route
        "reduce": dict(bytes=R * sh.K * by + 2.0 * sh.T * sh.K + 4.0 * R, flops=0.0,
                       name="moe_combine_kernel (top-k weighted reduction)", ncu="moe_combine_kernel"),
    }
    if small_batch_form(sh, small_batch):
        # the small-batch form: the same bytes and FLOPs in two warp-MMA kernels, then the same combine
        kern["gate_up"].update(name="moe_sb_up_kernel (gate/up + SwiGLU, warp MMA)", ncu="moe_sb_up_kernel")
        kern["down"].update(name="moe_sb_down_kernel (down + routing weight, warp MMA)", ncu="moe_sb_down_kernel")
    # the whole path's algorithmic HBM bytes: touched weights, x (+ its scales) read once, out written
    # once, the routing read, the planner's arrays written (sorted ids, expert ids, the padded total)
    cap = R + sh.E * (sh.block_m - 1)
    full = {"weights": bytes_w, "x": sh.T * sh.K * bx, "out": 2.0 * sh.T * sh.K, "routing": 8.0 * R,
            "plan": 4.0 * cap + 4.0 * ((cap + sh.block_m - 1) // sh.block_m) + 4.0}
    return dict(R=R, flops=flops, touched=touched, bytes_w=bytes_w, t_flop=t_flop, t_hbm=t_hbm,
                t_roof=max(t_flop, t_hbm), bound="tensor" if t_flop > t_hbm else "hbm", p_tc=p_tc, bw=bw,
                p1_bytes=kern["gate_up"]["bytes"], p1_flops=kern["gate_up"]["flops"], kernels=kern,
                bytes_full=sum(full.values()), bytes_parts=full)


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
    the current kernel source (the summary records the sha256 of the source
    file, csrc/fused_moe.cu unless it names another with ``source_file:``)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload_tag}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    f = re.search(r"source_file:\s*(\S+)", txt)
    if not m or not h:
        return None
    src = os.path.join(ROOT, "mixture_experts_ffn_planner_b200", "csrc", f.group(1) if f else "fused_moe.cu")
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != h.group(1):
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
def upload_weights(sh: W.Shape, inp: dict, dev) -> dict:
    """Host expert weights (the generator's arrays) to the device; e8m0 scales packed blocked."""
    import torch

    import mixture_experts_ffn_planner_b200 as moe

    def up(a, dtype=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(dtype) if dtype is not None else t).to(dev)

    if sh.dtype == "bf16":
        return dict(w1=up(inp["w1"], torch.bfloat16), w2=up(inp["w2"], torch.bfloat16), s1=None, s2=None)
    return dict(w1=up(inp["w1"]), w2=up(inp["w2"]), s1=moe.pack_scales_blocked(up(inp["w1_scales"])),
                s2=moe.pack_scales_blocked(up(inp["w2_scales"])))


def _expert_arrays(sh: W.Shape, which: str, e: int, seed: int):
    """One expert's weights as the caller hands them over: bf16 bits, or (codes, row-major scales)."""
    v = W.expert_f32(sh, which, e, seed)
    if sh.dtype == "bf16":
        return W.f32_to_bf16_bits(v), None
    return W.mx_quantize_fp4(v) if sh.dtype == "mxfp4" else W.mx_quantize_inputs(v)


def device_weights(sh: W.Shape, seed: int, dev, world: int = 1, rank: int = 0, dist=None, threads: int = 0) -> dict:
    """The workload's expert weights drawn expert by expert straight into device memory (no host copy
    of the whole set).  With several ranks each draws E/world of the experts and the ranks all-gather
    them, so every replica holds the same weights and the draws are split between the ranks."""
    import concurrent.futures as cf

    import torch

    import mixture_experts_ffn_planner_b200 as moe

    pack = 2 if sh.dtype == "mxfp4" else 1
    split = world > 1 and sh.E % world == 0
    lo, hi = (rank * sh.E // world, (rank + 1) * sh.E // world) if split else (0, sh.E)
    wdt = torch.uint16 if sh.dtype == "bf16" else torch.uint8
    dims = {"w1": (sh.N, sh.K), "w2": (sh.K, sh.I)}
    out = {}
    for which, (rows, cols) in dims.items():
        loc = torch.empty((hi - lo, rows, cols // pack), dtype=wdt, device=dev)
        sc = None if sh.dtype == "bf16" else torch.empty((hi - lo, rows, cols // 32), dtype=torch.uint8, device=dev)

        def job(e):
            v, s_ = _expert_arrays(sh, which, e, seed)
            loc[e - lo].copy_(torch.from_numpy(v))
            if sc is not None:
                sc[e - lo].copy_(torch.from_numpy(s_))
        n = threads if threads > 0 else max(1, min(32, (os.cpu_count() or 1) // max(1, world)))
        with cf.ThreadPoolExecutor(n) as ex:
            list(ex.map(job, range(lo, hi)))
        if split:
            full = torch.empty((sh.E,) + tuple(loc.shape[1:]), dtype=wdt, device=dev)
            dist.all_gather_into_tensor(full, loc)
            loc = full
            if sc is not None:
                fs = torch.empty((sh.E,) + tuple(sc.shape[1:]), dtype=torch.uint8, device=dev)
                dist.all_gather_into_tensor(fs, sc)
                sc = fs
        out[which] = loc.view(torch.bfloat16) if sh.dtype == "bf16" else loc
        out["s1" if which == "w1" else "s2"] = None if sc is None else moe.pack_scales_blocked(sc)
    return out


def step_inputs(sh: W.Shape, seed: int) -> dict:
    """A step's token batch: x (bf16 bits, or e4m3 codes + e8m0 scales) and the routing."""
    ids, tw = W.routing(sh, seed)
    d = dict(topk_ids=ids, topk_weights=tw)
    if sh.dtype == "bf16":
        d["x"] = W.f32_to_bf16_bits(W.x_f32(sh, seed))
    else:
        d["x"], d["x_scales"] = W.mx_quantize_inputs(W.x_f32(sh, seed))
    return d


def host_weights(sh: W.Shape, seed: int) -> dict:
    """The expert weights as host arrays (kept for the CPU oracle legs)."""
    if sh.dtype == "bf16":
        return dict(w1=W.bf16_weights(sh, "w1", seed), w2=W.bf16_weights(sh, "w2", seed))
    wq = W.mxfp4_weights if sh.dtype == "mxfp4" else W.mxfp8_weights
    w1, s1 = wq(sh, "w1", seed)
    w2, s2 = wq(sh, "w2", seed)
    return dict(w1=w1, w1_scales=s1, w2=w2, w2_scales=s2)


class Problem:
    """Device-resident inputs of one workload and one step of the hot path."""

    def __init__(self, sh: W.Shape, inp: dict, dev, stages: int = 0, ctas: int = 0, router: bool = False,
                 n_shared: int = 0, weights: dict | None = None, small_batch: int = 0):
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
        if weights is None:
            weights = upload_weights(sh, inp, dev)
        self.w1, self.w2, self.s1, self.s2 = weights["w1"], weights["w2"], weights["s1"], weights["s2"]
        if sh.dtype == "bf16":
            self.x = up(inp["x"], torch.bfloat16)
            self.xs = None
            dt = moe.DTYPE_BF16
        else:
            self.x, self.xs = up(inp["x"]), up(inp["x_scales"])
            dt = moe.DTYPE_MXFP4 if sh.dtype == "mxfp4" else moe.DTYPE_MXFP8
        self.ws = torch.empty(moe.moe_workspace_bytes(dt, sh.T, sh.K, sh.N, sh.E + n_shared, sh.top_k + n_shared, bm),
                              dtype=torch.uint8, device=dev)
        self.plain = moe.Tuning(stages, ctas, None)
        self.plain.small_batch = small_batch
        self.stages, self.ctas, self.small_batch = stages, ctas, small_batch
        # planner, gate/up phase, split-K reduction, down phase, combine (+ the router kernel for
        # batches of more than 32 tokens on the router path)
        # planner (+ router kernel beyond 32 tokens), then the four tensor-core launches or, for bf16
        # with few routed rows, the two small-batch kernels and the combine (the library's default switch)
        self.launches_per_step = (4 if small_batch_form(sh, small_batch) else 5) + (1 if router and sh.T > 32 else 0)

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


def graph_step_ms(prob: Problem, steps: int, flush=None):
    """Device time of one step replayed from a CUDA graph (the same library launches captured once),
    i.e. without the host's per-step submission through the Python binding; the L2 flush, when given,
    runs between replays outside the timed windows.  None if the capture is not possible here."""
    import torch

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.stream(stream):
            prob.step()  # the first call on this stream outside the capture
            with torch.cuda.graph(g, stream=stream):
                prob.step()
    except Exception:
        torch.cuda.synchronize()
        return None
    torch.cuda.current_stream().wait_stream(stream)
    cur = torch.cuda.current_stream()
    times = []
    for _ in range(3):
        g.replay()
    for _ in range(steps):
        if flush:
            flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        g.replay()
        e1.record(cur)
        times.append((e0, e1))
    torch.cuda.synchronize()
    prob.moe.moe_device_status()
    return float(np.median([a.elapsed_time(b) for a, b in times]))


def measure(prob: Problem, steps: int, warmup: int, flush_l2: bool = False, barrier=None, sample_clocks=True,
            local: int = 0, graph: bool = False):
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
    L2), reported beside the cold time and labelled as such.  With graph, the
    step is also captured once in a CUDA graph and replayed (median per step,
    same flush policy): the device-side time without per-step host submission.
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
    for t in tunes:
        t.small_batch = prob.small_batch
    timed(tunes, pev)
    moe.moe_device_status()
    warm_ms = None
    if flush_l2:
        prob.step()  # the last flush left L2 cold; one untimed step warms it
        warm_ms = timed(cold=False) / steps
        moe.moe_device_status()
    graph_ms = graph_step_ms(prob, steps, flush if flush_l2 else None) if graph else None
    return {"total_ms": total_ms, "ms_step": total_ms / steps, "warm_ms_step": warm_ms, "median_ms_step": median_ms,
            "graph_ms_step": graph_ms,
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


def roofline_of(sh: W.Shape, cm: dict, m: dict, peaks: dict, peak_src: str):
    """Roofline of the kernel with the longest device time in the step (pass 2 phase events):
    its algorithmic bytes (or FLOPs) per launch over its measured duration, against the measured
    HBM copy bandwidth (or the tensor peak of its MMA kind), whichever bound is slower."""
    phase_ms = {"gate_up": m["p1_ms"], "down": m["p2_ms"], "reduce": m["cb_ms"]}
    which = max(phase_ms, key=phase_ms.get)
    k = cm["kernels"][which]
    sec = phase_ms[which] * 1e-3
    tag = f"{sh.name}_T{sh.T}"
    pk_tc = tensor_peak(sh, peaks)
    base = {"kernel": k["name"], "phase": which, "us_per_launch": phase_ms[which] * 1e3,
            "share_of_step": phase_ms[which] / max(sum(phase_ms.values()) + m["plan_ms"], 1e-12),
            "traffic": kernel_traffic(k["ncu"], tag)}
    if k["flops"] / (pk_tc * 1e12) <= k["bytes"] / cm["bw"]:
        gbs = k["bytes"] / sec / 1e9
        return {**base, "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm_gbs",
                "algorithmic_bytes_per_launch": k["bytes"]}
    tf = k["flops"] / sec / 1e12
    src = f"{peak_src} bf16_tflops" if sh.dtype == "bf16" else \
        f"mxfp8 dense: {peaks.get('mxfp8_source', '2 x bf16 (nominal ratio)')}"
    return {**base, "bound": "tensor", "achieved": tf, "peak": pk_tc, "unit": "TFLOP/s", "frac": tf / pk_tc,
            "peak_source": src, "algorithmic_flops_per_launch": k["flops"]}


def result_line(sh, cm, m, world, steps, warmup, peaks, peak_src, flush_l2, small_batch: int = 0):
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
                   "tokens_per_gpu": sh.T, "parallelism": f"replicas x{world}", "l2": l2,
                   "form": "small-batch (warp MMA)" if small_batch_form(sh, small_batch) else "tcgen05 phases"},
        "us_per_call": ms_step * 1e3,
        **({"us_per_call_median": m["median_ms_step"] * 1e3} if m.get("median_ms_step") else {}),
        "weight_GBps": cm["bytes_w"] / (ms_step * 1e-3) / 1e9,
        "path_roofline": {"bound": cm["bound"], "t_roof_us": cm["t_roof"] * 1e6,
                          "frac": cm["t_roof"] / (ms_step * 1e-3), "touched_experts": cm["touched"],
                          "routed_gflop": cm["flops"] / 1e9, "touched_weight_gb": cm["bytes_w"] / 1e9,
                          "algorithmic_hbm_gb": cm["bytes_full"] / 1e9,
                          "algorithmic_hbm_parts_gb": {k: v / 1e9 for k, v in cm["bytes_parts"].items()},
                          "peaks": peak_src, "tensor_peak_tflops": tensor_peak(sh, peaks),
                          **({} if sh.dtype == "bf16" else
                             {"mxfp8_peak_source": peaks.get("mxfp8_source", "2 x bf16 (nominal ratio)")})},
        "phase_us": {"planner": m["plan_ms"] * 1e3, "gate_up": m["p1_ms"] * 1e3, "down": m["p2_ms"] * 1e3,
                     "reduce": m["cb_ms"] * 1e3},
        "roofline": roofline_of(sh, cm, m, peaks, peak_src),
        "gpu_launches": m["launches"],
        "clocks": m["clocks"],
        **({"graph": {"us_per_call_median": m["graph_ms_step"] * 1e3,
                      "note": "the same step captured once in a CUDA graph and replayed: device time without the "
                              "host's per-step submission (not the reported value)"}}
           if m.get("graph_ms_step") else {}),
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


def _setup_inputs(sh: W.Shape, args, rank: int, world: int, dist, dev, need_host: bool):
    """(shape with the shared experts, host inputs, device weights) of one workload.  Replicas share
    the expert weights (seed) and draw their own token batch (seed + rank)."""
    seed_w, seed_x = args.seed, args.seed + rank
    sh_w = dataclasses.replace(sh, E=sh.E + args.shared, top_k=sh.top_k + args.shared) if args.shared else sh
    inp = step_inputs(sh, seed_x)
    if args.shared:
        # the generator's routing over the routed experts, then the shared routes (cost model and
        # CPU baseline; the timed step routes from logits on the GPU)
        shared_ids = np.broadcast_to(np.arange(sh.E, sh.E + args.shared, dtype=np.int32), (sh.T, args.shared))
        inp["topk_ids"] = np.ascontiguousarray(np.concatenate([inp["topk_ids"], shared_ids], axis=1))
        inp["topk_weights"] = np.ascontiguousarray(
            np.concatenate([inp["topk_weights"], np.ones((sh.T, args.shared), np.float32)], axis=1))
    if args.router:
        inp["router_logits"], inp["router_bias"] = W.router_logits(sh, seed=seed_x)
    if need_host:
        inp.update(host_weights(sh_w, seed_w))
        weights = upload_weights(sh_w, inp, dev)
    else:
        weights = device_weights(sh_w, seed_w, dev, world, rank, dist)
    return sh_w, inp, weights


def bench_point(sh: W.Shape, sh_w: W.Shape, inp: dict, weights: dict, args, world: int, rank: int, local: int,
                dist, dev, peaks, peak_src, barrier, cpu_seconds: float):
    """Measures one workload and returns its JSON line (rank 0 prints it)."""
    cm = cost_model(sh_w, inp["topk_ids"], peaks, SMALL_BATCH_MODE[args.small_batch])
    prob = Problem(sh, inp, dev, args.stages, args.ctas, router=args.router, n_shared=args.shared, weights=weights,
                   small_batch=SMALL_BATCH_MODE[args.small_batch])
    flush = args.flush_l2 or cm["bytes_w"] < 4 * 126e6
    m = measure(prob, args.steps, args.warmup, flush_l2=flush, barrier=barrier, local=local,
                graph=world == 1 and not args.no_graph)
    m["ms_step"] = max_over_ranks(m["ms_step"], world, dist, dev)
    line = result_line(sh, cm, m, world, args.steps, args.warmup, peaks, peak_src, flush,
                       SMALL_BATCH_MODE[args.small_batch])
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
        rate, thr, desc, spent = oracle_sample_rate(sh_w, inp, cpu_seconds, args.seed, args.cpu_threads)
        line["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                "sample": desc, "seconds": spent}
    del prob
    return line


def _init(args):
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
    return world, rank, local, dist, torch.device("cuda", local)


def run_b200(args):
    world, rank, local, dist, dev = _init(args)
    barrier = dist.barrier if world > 1 else None
    peaks, peak_src = load_peaks()
    sh = W.shape(args.workload, args.tokens, **({"E": args.experts} if args.experts else {}))
    need_host = rank == 0 and world == 1 and not args.no_cpu_baseline
    sh_w, inp, weights = _setup_inputs(sh, args, rank, world, dist, dev, need_host)
    line = bench_point(sh, sh_w, inp, weights, args, world, rank, local, dist, dev, peaks, peak_src, barrier,
                       args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_sweep(args):
    """One line per (workload, token count) of the chosen configurations, on one GPU; every line
    carries its own clock record, path roofline, dominant-kernel roofline and CPU oracle sample
    (a shorter budget per line: --cpu-seconds / 5)."""
    import torch

    world, rank, local, dist, dev = _init(args)
    peaks, peak_src = load_peaks()
    for name in args.sweep_workloads.split(","):
        base = W.shape(name)
        weights = inp_w = None
        for T in W.token_counts(name):
            sh = W.shape(name, T)
            if weights is None:
                need_host = not args.no_cpu_baseline
                sh_w, inp, weights = _setup_inputs(sh, args, rank, world, dist, dev, need_host)
                inp_w = {k: v for k, v in inp.items() if k.startswith("w")}
            else:
                sh_w = sh
                inp = dict(step_inputs(sh, args.seed + rank), **inp_w)
                if args.router:
                    inp["router_logits"], inp["router_bias"] = W.router_logits(sh, seed=args.seed + rank)
            line = bench_point(sh, sh_w, inp, weights, args, world, rank, local, dist, dev, peaks, peak_src, None,
                               max(1.0, args.cpu_seconds / 5))
            line["sweep"] = f"{name} T={T}"
            print(json.dumps(line), flush=True)
        del weights, inp_w, base
        torch.cuda.empty_cache()
    return 0


def run_peak(args):
    """Dense tensor-core peaks on this GPU: a bf16 GEMM (torch.matmul) and an mxfp8 GEMM
    (torch.nn.functional.scaled_mm, e4m3 operands with one e8m0 scale per 32 along K), both
    M = N = K = 8192, as a burst (best of 20 timed calls) and sustained (back to back for ~4 s)."""
    import torch
    import torch.nn.functional as F

    _, _, local, _, dev = _init(args)
    n = 8192
    flop = 2.0 * n ** 3
    a16 = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    b16 = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    a8 = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b8 = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    ones = torch.full((n * n // 32,), 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)

    def mx():
        return F.scaled_mm(a8, b8.t(), ones, F.ScalingType.BlockWise1x32, ones, F.ScalingType.BlockWise1x32,
                           swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                           output_dtype=torch.bfloat16)

    def bf():
        return a16 @ b16

    res = {"metric": "dense tensor-core peak", "M=N=K": n}
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    for name, fn in (("bf16", bf), ("mxfp8", mx)):
        try:
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            best = float("inf")
            for _ in range(20):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                best = min(best, e0.elapsed_time(e1))
            t0 = time.perf_counter()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            calls = 0
            while time.perf_counter() - t0 < 4.0:
                for _ in range(20):
                    fn()
                calls += 20
                torch.cuda.synchronize()
            e1.record()
            torch.cuda.synchronize()
            res[f"{name}_tflops_burst"] = flop / (best * 1e-3) / 1e12
            res[f"{name}_tflops_sustained"] = flop * calls / (e0.elapsed_time(e1) * 1e-3) / 1e12
        except Exception as exc:  # an operand type this torch build cannot run
            res[f"{name}_error"] = f"{type(exc).__name__}: {exc}"[:300]
    res["clocks"] = clocks.stop()
    print(json.dumps(res), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.peak:
        return run_peak(args)
    if args.sweep:
        return run_sweep(args)
    return run_b200(args)


if __name__ == "__main__":
    sys.exit(main())
