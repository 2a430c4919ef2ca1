"""moe_route_align on the GPU against the oracle.

The router (softmax over the experts, top-k, renormalised weights; "Prime Flash MoE",
Usage and "[RFC] Fused W8A8 MoE megakernel on H20", Results so far) decides integer ids
from fp32 scores, which both sides form the same way (one fp32 addition of logit and
bias), so topk_ids must be bit-exact; the weights are fp32 on the GPU against the
oracle's float64 (|diff| <= 2e-6, a few fp32 ulps of values <= 1).  The planner outputs
that follow must equal the oracle planner's on the oracle's ids, bit for bit.  Batches of
at most 32 tokens take the in-planner router, larger ones the all-SM router kernel; both
are covered, at the workloads' sizes and at the edges.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import to_dev

pytestmark = pytest.mark.gpu

W_TOL = 2e-6


def _run(logits: np.ndarray, bias, k: int, bm: int, S: int = 0):
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    T, E = logits.shape
    cap = moe.moe_align_capacity(T, k + S, E + S, bm)
    d_logits = to_dev(logits) if logits.size else torch.empty((T, E), dtype=torch.float32, device="cuda")
    d_bias = None if bias is None else to_dev(bias)
    # poisoned outputs: any element the kernels skip shows up
    ids = torch.full((T, k + S), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    w = torch.full((T, k + S), float("nan"), dtype=torch.float32, device="cuda")
    s = torch.full((cap,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    e = torch.full(((cap + bm - 1) // bm,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    n = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    moe.moe_route_align(d_logits, k, bm, d_bias, ids, w, s, e, n, n_shared=S)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy(), s.cpu().numpy(), e.cpu().numpy(), int(n.cpu().numpy()[0])


def _check(logits, bias, k, bm, S=0):
    T, E = logits.shape
    rid, rw = oracle.route_topk(logits, k, bias, n_shared=S)
    gid, gw, gs, ge, gn = _run(logits, bias, k, bm, S)
    np.testing.assert_array_equal(gid, rid)
    assert np.all(np.abs(gw.astype(np.float64) - rw) <= W_TOL), float(np.max(np.abs(gw - rw)))
    rs, re_, rn = oracle.moe_align(rid, E + S, bm)
    assert gn == rn
    np.testing.assert_array_equal(gs, rs)
    np.testing.assert_array_equal(ge, re_)


@pytest.mark.parametrize("name,T", [("C1", 64), ("C2", 64), ("C2", 256), ("C3", 64), ("C3", 1024), ("C3", 8192),
                                    ("C4", 2048), ("C5", 1), ("C5", 8), ("C5", 64), ("C5", 512), ("C5", 8192)])
def test_workloads(name, T):
    sh = W.shape(name, T)
    logits, bias = W.router_logits(sh)
    _check(logits, bias, sh.top_k, sh.block_m)


@pytest.mark.parametrize("T", [0, 1, 31, 32, 33, 300])   # both sides of the in-planner limit (32)
@pytest.mark.parametrize("E,k", [(1, 1), (9, 3), (256, 8), (1024, 8), (33, 8)])
def test_sizes(T, E, k):
    rng = np.random.default_rng(T * 17 + E * 3 + k)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = rng.standard_normal(E).astype(np.float32) if E % 2 else None
    _check(logits, bias, k, 64)


@pytest.mark.parametrize("T", [20, 1000])
def test_ties_go_to_the_lower_index(T):
    # scores on a coarse grid: many exact ties inside every row, and between a row's
    # top-k boundary and the experts just outside it
    rng = np.random.default_rng(T)
    logits = (rng.integers(-3, 3, size=(T, 40)) * 0.5).astype(np.float32)
    _check(logits, None, 8, 32)
    _check(np.zeros((T, 40), np.float32), None, 8, 32)   # all equal: experts 0..7, weights 1/8


def test_routed_ids_drive_the_ffn():
    # the whole path from router logits: route + plan, then the bf16 FFN, on the GPU; the
    # oracle side routes with its own router (no oracle input comes from the CUDA path)
    import torch
    import mixture_experts_ffn_planner_b200 as moe
    from tests.helpers import assert_bf16_parity, out_bits

    sh = W.shape("C1", 64)
    inp = W.inputs(sh)
    logits, bias = W.router_logits(sh)
    _, d_w, s, e, n = moe.moe_route_align(to_dev(logits), sh.top_k, sh.block_m,
                                          None if bias is None else to_dev(bias))
    x, w1, w2 = (to_dev(inp[k], torch.bfloat16) for k in ("x", "w1", "w2"))
    out = torch.full((sh.T, sh.K), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.fused_moe_bf16(x, w1, w2, s, e, n, d_w, out, sh.block_m)
    moe.moe_device_status()
    got = out_bits(out)
    rid, rw = oracle.route_topk(logits, sh.top_k, bias)
    ref = oracle.fused_moe_bf16(inp["x"], inp["w1"], inp["w2"], rid, rw.astype(np.float32), unrounded=True)[1]
    assert_bf16_parity(got, ref, "routed C1")


@pytest.mark.parametrize("T", [8, 32, 300])
@pytest.mark.parametrize("S", [1, 2])
def test_shared_experts(T, S):
    rng = np.random.default_rng(T * 7 + S)
    _check(rng.standard_normal((T, 64)).astype(np.float32), None, 6, 64, S)
    sh = W.shape("C3", 64)
    logits, bias = W.router_logits(sh)
    _check(logits[:T] if T <= 64 else np.tile(logits, (5, 1))[:T], bias, sh.top_k, sh.block_m, S)


@pytest.mark.parametrize("dtype", ["bf16", "mxfp8"])
def test_shared_expert_in_the_fused_kernels(dtype):
    """Routed experts plus one shared expert (stored after them) in one fused call, against
    the oracle routing with its own router and running the FFN on E + 1 experts."""
    import torch
    import mixture_experts_ffn_planner_b200 as moe
    from tests.helpers import assert_bf16_parity, assert_mxfp8_parity, out_bits

    E, S, k, T, K, N, bm = 8, 1, 2, 200, 256, 512, 64
    sh = W.Shape(name="S", dtype=dtype, T=T, K=K, N=N, E=E + S, top_k=k + S, block_m=bm, zipf_s=None)
    inp = W.inputs(sh, seed=5)                  # x and the weights of E + S experts
    logits = np.random.default_rng(6).standard_normal((T, E)).astype(np.float32)
    _, d_w, s_ids, e_ids, ntpp = moe.moe_route_align(to_dev(logits), k, bm, None, n_shared=S)
    out = torch.full((T, K), float("nan"), dtype=torch.bfloat16, device="cuda")
    rid, rw = oracle.route_topk(logits, k, None, n_shared=S)
    if dtype == "bf16":
        x, w1, w2 = (to_dev(inp[n], torch.bfloat16) for n in ("x", "w1", "w2"))
        moe.fused_moe_bf16(x, w1, w2, s_ids, e_ids, ntpp, d_w, out, bm)
        ref = oracle.fused_moe_bf16(inp["x"], inp["w1"], inp["w2"], rid, rw.astype(np.float32), unrounded=True)[1]
        check = assert_bf16_parity
    else:
        x, xs, w1, w2 = (to_dev(inp[n]) for n in ("x", "x_scales", "w1", "w2"))
        s1 = moe.pack_scales_blocked(to_dev(inp["w1_scales"]))
        s2 = moe.pack_scales_blocked(to_dev(inp["w2_scales"]))
        moe.fused_moe_mxfp8(x, xs, w1, s1, w2, s2, s_ids, e_ids, ntpp, d_w, out, bm)
        ref = oracle.fused_moe_mxfp8(inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], inp["w2"],
                                     inp["w2_scales"], rid, rw.astype(np.float32), unrounded=True)[1]
        check = assert_mxfp8_parity
    moe.moe_device_status()
    check(out_bits(out), ref, f"{dtype} with a shared expert")
