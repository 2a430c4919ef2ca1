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

Multi-GPU: ``torchrun --nproc-per-node N bench.py --gpus N``; every rank is an
independent replica with all experts resident (no collective on the data
path); time is the max over ranks, ``value`` the sum of all ranks' work.
"""
from __future__ import annotations

import argparse
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
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default="C2", choices=W.workload_names())
    ap.add_argument("--tokens", type=int, default=256)
    ap.add_argument("--seed", type=int, default=W.DEFAULT_SEED)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the CPU oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--stages", type=int, default=0)
    ap.add_argument("--ctas", type=int, default=0)
    return ap.parse_args(argv)


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
    b = 2.0 if sh.dtype == "bf16" else 1.0 + 1.0 / 32.0
    bytes_w = touched * 1.5 * sh.N * sh.K * b
    p_tc = peaks["bf16_tflops"] * (1.0 if sh.dtype == "bf16" else 2.0) * 1e12
    bw = peaks["hbm_gbs"] * 1e9
    t_flop, t_hbm = flops / p_tc, bytes_w / bw
    # gate/up phase: w1 of the touched experts, the routed rows of x, the intermediate written once
    bx = 2.0 if sh.dtype == "bf16" else 1.0 + 1.0 / 32.0
    p1_bytes = touched * sh.N * sh.K * b + R * sh.K * bx + R * sh.I * bx
    p1_flops = 2.0 * R * sh.K * sh.N
    return dict(R=R, flops=flops, touched=touched, bytes_w=bytes_w, t_flop=t_flop, t_hbm=t_hbm,
                t_roof=max(t_flop, t_hbm), bound="tensor" if t_flop > t_hbm else "hbm", p_tc=p_tc, bw=bw,
                p1_bytes=p1_bytes, p1_flops=p1_flops)


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
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


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
def oracle_sample_rate(sh: W.Shape, inp: dict, seconds: float, seed: int):
    """Times the oracle on a growing token sample until ~`seconds` of work; returns
    (TFLOP/s, threads, description)."""
    import oracle

    thr = os.cpu_count() or 1
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
    return oracle.fused_moe_mxfp8(inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], inp["w2"],
                                  inp["w2_scales"], inp["topk_ids"], inp["topk_weights"], tokens=toks, nthreads=thr)


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sh = W.shape(args.workload, args.tokens)
    inp = W.inputs(sh, seed=args.seed)
    thr = os.cpu_count() or 1
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
def run_b200(args):
    import torch
    import torch.distributed as dist

    import mixture_experts_ffn_planner_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()

    sh = W.shape(args.workload, args.tokens)
    inp = W.inputs(sh, seed=args.seed + rank)  # every replica gets its own batch
    cm = cost_model(sh, inp["topk_ids"], peaks)

    def up(a, dtype=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(dtype) if dtype is not None else t).to(dev)

    ids, tw = up(inp["topk_ids"]), up(inp["topk_weights"])
    bm = sh.block_m
    cap = moe.moe_align_capacity(sh.T, sh.top_k, sh.E, bm)
    s_ids = torch.empty(cap, dtype=torch.int32, device=dev)
    e_ids = torch.empty((cap + bm - 1) // bm, dtype=torch.int32, device=dev)
    ntpp = torch.empty(1, dtype=torch.int32, device=dev)
    out = torch.empty((sh.T, sh.K), dtype=torch.bfloat16, device=dev)
    if sh.dtype == "bf16":
        x, w1, w2 = up(inp["x"], torch.bfloat16), up(inp["w1"], torch.bfloat16), up(inp["w2"], torch.bfloat16)
        ws = torch.empty(moe.moe_workspace_bytes(moe.DTYPE_BF16, sh.T, sh.K, sh.N, sh.E, sh.top_k, bm),
                         dtype=torch.uint8, device=dev)

        def fused(tune):
            moe.fused_moe_bf16(x, w1, w2, s_ids, e_ids, ntpp, tw, out, bm, workspace=ws, tune=tune)
    else:
        x, xs, w1, w2 = up(inp["x"]), up(inp["x_scales"]), up(inp["w1"]), up(inp["w2"])
        s1 = moe.pack_scales_blocked(up(inp["w1_scales"]))
        s2 = moe.pack_scales_blocked(up(inp["w2_scales"]))
        ws = torch.empty(moe.moe_workspace_bytes(moe.DTYPE_MXFP8, sh.T, sh.K, sh.N, sh.E, sh.top_k, bm),
                         dtype=torch.uint8, device=dev)

        def fused(tune):
            moe.fused_moe_mxfp8(x, xs, w1, s1, w2, s2, s_ids, e_ids, ntpp, tw, out, bm, workspace=ws, tune=tune)

    stream = torch.cuda.current_stream()
    n_ev = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_ev)]
    tunes = [moe.Tuning.with_events(e, args.stages, args.ctas) for e in ev]
    plain = moe.Tuning(args.stages, args.ctas, None)

    def step(tune):
        moe.moe_align(ids, sh.E, bm, s_ids, e_ids, ntpp)
        fused(tune)

    for _ in range(max(3, args.warmup)):
        step(plain)
    moe.moe_device_status()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(tunes[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    moe.moe_device_status()
    ms_local = t_start.elapsed_time(t_end)
    p1_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    p2_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    cb_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    ms = ms_local
    if world > 1:
        t = torch.tensor([ms_local], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    ms_step = ms / args.steps
    value = world * cm["flops"] / (ms_step * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        hx = torch.from_numpy(np.ascontiguousarray(inp["x"]))
        hx = hx.view(torch.bfloat16) if sh.dtype == "bf16" else hx
        host_in = [hx.pin_memory(), torch.from_numpy(inp["topk_ids"]).pin_memory(),
                   torch.from_numpy(inp["topk_weights"]).pin_memory()]
        if sh.dtype == "mxfp8":
            host_in.append(torch.from_numpy(np.ascontiguousarray(inp["x_scales"])).pin_memory())
        dev_in = [x, ids, tw] + ([xs] if sh.dtype == "mxfp8" else [])
        host_out = torch.empty((sh.T, sh.K), dtype=torch.bfloat16).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = host_out.numel() * host_out.element_size()
        for _ in range(3):
            for h, d in zip(host_in, dev_in):
                d.copy_(h, non_blocking=True)
            step(plain)
            host_out.copy_(out, non_blocking=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            for h, d in zip(host_in, dev_in):
                d.copy_(h, non_blocking=True)
            step(plain)
            host_out.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1)
        if world > 1:
            t = torch.tensor([ems], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        e2e = {"value": world * cm["flops"] / (ems / args.steps * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "us_per_call": 1e3 * ems / args.steps}

    # ---- dominant kernel (gate/up phase) against its roofline
    p1_s = p1_ms * 1e-3
    p1_tflops = cm["p1_flops"] / p1_s / 1e12
    p1_gbs = cm["p1_bytes"] / p1_s / 1e9
    p1_bound = "tensor" if cm["p1_flops"] / cm["p_tc"] > cm["p1_bytes"] / cm["bw"] else "hbm"
    tag = f"{sh.name}_T{sh.T}"
    if p1_bound == "hbm":
        roof = {"kernel": "moe_p1_kernel (gather + gate/up GEMM + SwiGLU)", "bound": "hbm", "achieved": p1_gbs,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": p1_gbs / peaks["hbm_gbs"],
                "traffic": kernel_traffic("moe_p1_kernel", tag), "peak_source": f"{peak_src} hbm_gbs",
                "algorithmic_bytes_per_launch": cm["p1_bytes"], "us_per_launch": p1_ms * 1e3}
    else:
        pk = peaks["bf16_tflops"] * (1.0 if sh.dtype == "bf16" else 2.0)
        roof = {"kernel": "moe_p1_kernel (gather + gate/up GEMM + SwiGLU)", "bound": "tensor",
                "achieved": p1_tflops, "peak": pk, "unit": "TFLOP/s", "frac": p1_tflops / pk,
                "traffic": kernel_traffic("moe_p1_kernel", tag),
                "peak_source": f"{peak_src} bf16_tflops" + ("" if sh.dtype == "bf16" else " x 2 (fp8:bf16 nominal)"),
                "algorithmic_flops_per_launch": cm["p1_flops"], "us_per_launch": p1_ms * 1e3}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": sh.dtype, "data": "synthetic (seeded workloads generator, random weights)",
        "config": {"workload": f"{sh.name}: {sh.dtype} MoE FFN K={sh.K} N={sh.N} (intermediate {sh.I}) "
                               f"E={sh.E} top_k={sh.top_k} T={sh.T} block_m={bm}",
                   "tokens_per_gpu": sh.T, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2 (touched expert weights {cm['bytes_w'] / 1e9:.2f} GB per step)"},
        "us_per_call": ms_step * 1e3,
        "weight_GBps": cm["bytes_w"] / (ms_step * 1e-3) / 1e9,
        "path_roofline": {"bound": cm["bound"], "t_roof_us": cm["t_roof"] * 1e6, "frac": cm["t_roof"] / (ms_step * 1e-3),
                          "touched_experts": cm["touched"], "routed_gflop": cm["flops"] / 1e9,
                          "touched_weight_gb": cm["bytes_w"] / 1e9, "peaks": peak_src},
        "phase_us": {"gate_up": p1_ms * 1e3, "down": p2_ms * 1e3, "reduce": cb_ms * 1e3},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, thr, desc, spent = oracle_sample_rate(sh, inp, args.cpu_seconds, args.seed)
        line["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                "sample": desc, "seconds": spent}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del tunes
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
