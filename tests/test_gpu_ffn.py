"""Fused MoE forward on the GPU (planner + fused kernels, through the C ABI)
against the oracle on the same seeded inputs.

bf16 path: max|gpu - oracle| <= 2e-2 * rms(oracle out).
mxfp8 path (the oracle emulates the on-chip requant): cosine >= 0.999 and
max|gpu - oracle| <= 6e-2 * rms(oracle out).  "oracle out" is the oracle's
result before its final rounding to bf16 (see tests/helpers.py).
Small cases run the whole oracle; they span several 128-row blocks, several
intermediate tiles and a ragged tail.  The named workloads at full size run
the whole oracle up to 256 tokens and otherwise a seeded sample of 512 tokens
(tokens are independent, so their rows are exact sub-results) that covers
every non-empty expert, the last row of full blocks and the last block
(tests/helpers.coverage_sample).
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_bf16_parity, assert_mxfp8_parity, coverage_sample, out_bits, to_dev

FULL_SAMPLE = 512  # tokens compared at full size (the whole batch when it is smaller)

pytestmark = pytest.mark.gpu


def gpu_forward(sh: W.Shape, inp: dict, block_m: int | None = None, tune=None, repeat: int = 1):
    """Uploads the inputs, runs moe_align + fused_moe_*; returns host bf16 bits (T, K) per repeat."""
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    bm = block_m or sh.block_m
    ids = to_dev(inp["topk_ids"])
    tw = to_dev(inp["topk_weights"])
    sorted_ids, expert_ids, ntpp = moe.moe_align(ids, sh.E, bm)
    outs = []
    if sh.dtype == "bf16":
        x, w1, w2 = (to_dev(inp[n], torch.bfloat16) for n in ("x", "w1", "w2"))
        for _ in range(repeat):
            out = torch.full((sh.T, sh.K), float("nan"), dtype=torch.bfloat16, device="cuda")
            moe.fused_moe_bf16(x, w1, w2, sorted_ids, expert_ids, ntpp, tw, out, bm, tune=tune)
            outs.append(out)
    else:
        x, xs, w1, w2 = (to_dev(inp[n]) for n in ("x", "x_scales", "w1", "w2"))
        s1 = moe.pack_scales_blocked(to_dev(inp["w1_scales"]))
        s2 = moe.pack_scales_blocked(to_dev(inp["w2_scales"]))
        fwd = moe.fused_moe_mxfp4 if sh.dtype == "mxfp4" else moe.fused_moe_mxfp8
        for _ in range(repeat):
            out = torch.full((sh.T, sh.K), float("nan"), dtype=torch.bfloat16, device="cuda")
            fwd(x, xs, w1, s1, w2, s2, sorted_ids, expert_ids, ntpp, tw, out, bm, tune=tune)
            outs.append(out)
    moe.moe_device_status()
    res = [out_bits(o) for o in outs]
    return res if repeat > 1 else res[0]


def oracle_forward(sh: W.Shape, inp: dict, tokens=None):
    """The oracle's out before its final bf16 rounding (float64, (T, K))."""
    if sh.dtype == "bf16":
        return oracle.fused_moe_bf16(inp["x"], inp["w1"], inp["w2"], inp["topk_ids"], inp["topk_weights"],
                                     tokens=tokens, unrounded=True)[1]
    fwd = oracle.fused_moe_mxfp4 if sh.dtype == "mxfp4" else oracle.fused_moe_mxfp8
    return fwd(inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], inp["w2"], inp["w2_scales"],
               inp["topk_ids"], inp["topk_weights"], tokens=tokens, unrounded=True)[1]


def check(sh, got, ref, what):
    if sh.dtype == "bf16":
        return assert_bf16_parity(got, ref, what)
    return assert_mxfp8_parity(got, ref, what)


def small(dtype, T, K, N, E, top_k, block_m, zipf=None):
    return W.Shape(name="S", dtype=dtype, T=T, K=K, N=N, E=E, top_k=top_k, block_m=block_m, zipf_s=zipf)


SMALL_BF16 = [
    small("bf16", 200, 256, 512, 8, 2, 128),      # 2 intermediate tiles, ragged blocks
    small("bf16", 200, 256, 512, 8, 2, 64),
    small("bf16", 77, 128, 320, 5, 3, 32),        # I = 160: partial intermediate tile
    small("bf16", 50, 384, 80, 6, 2, 16),         # I = 40: partial 64-wide K chunk in the down GEMM
    small("bf16", 300, 256, 256, 16, 4, 128, 1.2),  # skewed routing, empty experts
    small("bf16", 1, 128, 256, 4, 1, 128),
    small("bf16", 12, 1024, 512, 4, 2, 64),       # few units, few rows: split-K (8 splits)
    small("bf16", 10, 512, 320, 3, 2, 32),        # split-K with a partial intermediate tile (I = 160)
]
SMALL_MXFP8 = [
    small("mxfp8", 200, 256, 512, 8, 2, 128),
    small("mxfp8", 200, 512, 256, 8, 2, 64),
    small("mxfp8", 90, 256, 768, 6, 3, 32),       # I = 384: 3 intermediate tiles
    small("mxfp8", 300, 256, 256, 16, 4, 128, 1.2),
    small("mxfp8", 12, 1024, 512, 4, 2, 128),     # split-K (4 splits)
]
SMALL_MXFP4 = [                                    # MXFP4 weights, mxfp8 activations
    small("mxfp4", 200, 256, 512, 8, 2, 128),
    small("mxfp4", 200, 512, 256, 8, 2, 64),
    small("mxfp4", 90, 256, 768, 6, 3, 32),
    small("mxfp4", 300, 256, 256, 16, 4, 128, 1.2),
    small("mxfp4", 12, 1024, 512, 4, 2, 128),     # split-K
    small("mxfp4", 1, 256, 256, 3, 1, 16),
]


@pytest.mark.parametrize("sh", SMALL_BF16 + SMALL_MXFP8 + SMALL_MXFP4, ids=lambda s: f"{s.dtype}-T{s.T}-K{s.K}-N{s.N}-E{s.E}-"
                         f"k{s.top_k}-bm{s.block_m}")
def test_small_full_oracle(sh):
    inp = W.inputs(sh, seed=11)
    got = gpu_forward(sh, inp)
    ref = oracle_forward(sh, inp)
    check(sh, got, ref, "small")


@pytest.mark.parametrize("dtype", ["bf16", "mxfp8"])
@pytest.mark.parametrize("T", [300, 12])  # 12 tokens: the split-K path
def test_deterministic(dtype, T):
    sh = small(dtype, T, 1024 if T < 100 else 256, 512, 8, 3, 128)
    a, b = gpu_forward(sh, W.inputs(sh, seed=3), repeat=2)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("dtype", ["bf16", "mxfp8"])
def test_invalid_routes_contribute_nothing(dtype):
    """Routes whose expert id is outside [0, E) get no slot and add nothing."""
    sh = small(dtype, 64, 256, 256, 4, 2, 128)
    inp = W.inputs(sh, seed=4)
    inp["topk_ids"] = inp["topk_ids"].copy()
    inp["topk_ids"][::3, 1] = -1
    inp["topk_ids"][5, :] = 9
    got = gpu_forward(sh, inp)
    ref = oracle_forward(sh, inp)
    check(sh, got, ref, "invalid ids")
    assert not got[5].any() or np.all((got[5] & 0x7FFF) == 0)


@pytest.mark.parametrize("stages", [2, 3])
def test_tuning_stages(stages):
    import mixture_experts_ffn_planner_b200 as moe

    sh = small("bf16", 150, 512, 512, 8, 2, 128)
    inp = W.inputs(sh, seed=8)
    got = gpu_forward(sh, inp, tune=moe.Tuning(stages=stages, num_ctas=7))
    check(sh, got, oracle_forward(sh, inp), f"stages={stages}")


def test_c1_full():
    """bf16, T=64, K=1024, N=1024, E=8, top-2, block_m=64: whole oracle."""
    sh = W.shape("C1", 64)
    inp = W.inputs(sh)
    rel, cos = check(sh, gpu_forward(sh, inp), oracle_forward(sh, inp), "C1")
    print(f"PARITY C1 T=64 tokens=64 max|diff|/rms={rel:.3e} cos={cos:.7f}")


@pytest.mark.parametrize("T", [1, 8, 64, 512, 8192])
def test_c5(T):
    """bf16 narrow intermediate with Zipf-skewed routing (empty experts): whole batch up to T=512,
    a 512-token coverage sample at T=8192."""
    sh = W.shape("C5", T)
    inp = W.inputs(sh)
    toks = coverage_sample(sh, inp["topk_ids"], FULL_SAMPLE)
    got = gpu_forward(sh, inp)
    ref = oracle_forward(sh, inp, tokens=toks)
    rel, cos = check(sh, got[toks], ref[toks], f"C5 T={T}")
    print(f"PARITY C5 T={T} tokens={len(toks)} max|diff|/rms={rel:.3e} cos={cos:.7f}")


# ---------------------------------------------------------------- full-size workloads, sampled tokens
_WEIGHTS = {}


def _weights(name):
    """Expert weights of a named workload, generated once per test session."""
    if name not in _WEIGHTS:
        _WEIGHTS.clear()  # hold one workload's weights at a time (C4 is ~26 GB in mxfp8)
        sh = W.shape(name)
        if sh.dtype == "bf16":
            _WEIGHTS[name] = dict(w1=W.bf16_weights(sh, "w1"), w2=W.bf16_weights(sh, "w2"))
        else:
            wq = W.mxfp4_weights if sh.dtype == "mxfp4" else W.mxfp8_weights
            w1, s1 = wq(sh, "w1")
            w2, s2 = wq(sh, "w2")
            _WEIGHTS[name] = dict(w1=w1, w1_scales=s1, w2=w2, w2_scales=s2)
    return _WEIGHTS[name]


def _full_inputs(name, T):
    sh = W.shape(name, T)
    ids, tw = W.routing(sh)
    inp = dict(_weights(name), topk_ids=ids, topk_weights=tw)
    if sh.dtype == "bf16":
        inp["x"] = W.f32_to_bf16_bits(W.x_f32(sh))
    else:
        inp["x"], inp["x_scales"] = W.mx_quantize_inputs(W.x_f32(sh))
    return sh, inp


FULL_CASES = [("C2", 64), ("C2", 256),
              ("C3", 64), ("C3", 256), ("C3", 1024), ("C3", 2048), ("C3", 4096), ("C3", 8192),
              ("C4", 1024), ("C4", 2048), ("C4", 4096), ("C4", 8192),
              ("C3F4", 64), ("C3F4", 2048), ("C3F4", 8192),
              ("C4F4", 1024), ("C4F4", 8192)]


@pytest.mark.parametrize("name,T", FULL_CASES)
def test_full_size(name, T):
    """The workload at full size through the GPU path; parity on the whole batch (T <= 256) or a
    512-token coverage sample (every non-empty expert, block tails, the last block)."""
    sh, inp = _full_inputs(name, T)
    toks = coverage_sample(sh, inp["topk_ids"], FULL_SAMPLE)
    got = gpu_forward(sh, inp)
    ref = oracle_forward(sh, inp, tokens=toks)
    rel, cos = check(sh, got[toks], ref[toks], f"{name} T={T}")
    assert np.isfinite(W.bf16_bits_to_f32(got)).all()
    print(f"PARITY {name} T={T} tokens={len(toks)} experts={len(np.unique(inp['topk_ids'][toks]))} "
          f"max|diff|/rms={rel:.3e} cos={cos:.7f}")
